"""Backward pass on the GPU against the fp64 oracle's backward, itself pinned to
central finite differences of the forward rule.  Every case runs both
algorithms: the chunk form (gdn_prefill_backward with its full workspace) and
the sequential one (gdn_prefill_backward_sequential)."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_recurrence_rule_b200 import api, inputs
from parity import o_error, to_np

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
TOL = 1e-4  # fp32 arithmetic against fp64 on the same inputs: max|err| / RMS(ref) per gradient


@pytest.fixture(params=["chunked", "sequential"])
def algo(request):
    return request.param


def _case(lengths, Hqk, Hv, D, dtype, seed, algo, init=True, dsf=True, scale=0.5, edit=None):
    inp = inputs.prefill_inputs(lengths, Hqk, Hv, D, dtype=dtype, seed=seed,
                                init_std=0.1 if init else 0.0)
    if edit is not None:
        edit(inp)
    T, N = sum(lengths), len(lengths)
    gen = torch.Generator().manual_seed(seed + 700)
    d_o = torch.randn(T, Hv, D, generator=gen)
    d_sf = torch.randn(N, Hv, D, D, generator=gen) * 0.1 if dsf else None
    dev = {n: (t.to(DEV) if t is not None else None) for n, t in inp.items()}
    out = api.prefill_backward(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], d_o.to(DEV),
                               cu_seqlens=dev["cu_seqlens"], initial_state=dev["initial_state"],
                               d_final_state=None if d_sf is None else d_sf.to(DEV), scale=scale,
                               sequential=algo == "sequential")
    torch.cuda.synchronize()
    ref = oracle.backward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], d_o,
                          cu_seqlens=inp["cu_seqlens"], initial_state=inp["initial_state"],
                          d_final_state=d_sf, scale=scale)
    return out, ref


def _check(out, ref, what):
    for name, a, b in zip(("dq", "dk", "dv", "dg", "dbeta", "ds0"), out, ref):
        a = to_np(a)
        assert np.isfinite(a).all(), f"{what}: non-finite {name}"
        e = o_error(a, b)
        assert e <= TOL, f"{what}: {name} max|err|/RMS = {e:.3e} > {TOL:.0e}"


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
def test_backward_varlen_gqa(dtype, D, algo):
    out, ref = _case([37, 0, 50, 16], 2, 6, D, dtype, seed=101 + D, algo=algo)
    _check(out, ref, f"{algo} {dtype} D={D}")


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_backward_chunk_boundaries(dtype, algo):
    """Sequences of exactly one chunk, one chunk plus a token, two chunks plus
    one, a single token and several chunks with a ragged tail, at D=128."""
    out, ref = _case([64, 65, 129, 1, 200], 2, 6, 128, dtype, seed=121, algo=algo)
    _check(out, ref, f"{algo} {dtype} chunk boundaries")


def test_backward_degenerate_gates(algo):
    """alpha = 0 (g = -inf) on single tokens, at the first and last token of a
    16-token checkpoint interval and on a run; g = 0 on a stretch; beta = 0 and
    beta = 1 on others."""
    def edit(inp):
        inp["g"][[0, 5, 15, 16, 17, 18, 60, 75]] = -float("inf")
        inp["g"][30:45] = 0.0
        inp["beta"][[3, 4, 50, 80]] = 0.0
        inp["beta"][[7, 33, 90]] = 1.0
    out, ref = _case([70, 40], 2, 6, 64, "fp32", seed=111, algo=algo, edit=edit)
    _check(out, ref, f"{algo} gates")


def test_backward_mixed_dims(algo):
    """Dk != Dv, one value head per query/key head (dq, dk written directly)."""
    for Dk, Dv in ((128, 64), (64, 128)):
        inp = inputs.prefill_inputs([40, 23], 2, 2, Dk, dtype="fp32", seed=105, init_std=0.1)
        gen = torch.Generator().manual_seed(106)
        T = 63
        v = torch.randn(T, 2, Dv, generator=gen)
        s0 = torch.randn(2, 2, Dv, Dk, generator=gen) * 0.1
        d_o = torch.randn(T, 2, Dv, generator=gen)
        out = api.prefill_backward(inp["q"].to(DEV), inp["k"].to(DEV), v.to(DEV), inp["g"].to(DEV),
                                   inp["beta"].to(DEV), d_o.to(DEV),
                                   cu_seqlens=inp["cu_seqlens"].to(DEV), initial_state=s0.to(DEV),
                                   sequential=algo == "sequential")
        torch.cuda.synchronize()
        ref = oracle.backward(inp["q"], inp["k"], v, inp["g"], inp["beta"], d_o,
                              cu_seqlens=inp["cu_seqlens"], initial_state=s0)
        _check(out, ref, f"{algo} Dk={Dk} Dv={Dv}")


@pytest.mark.parametrize("Dk,Dv", [(128, 64), (64, 128)])
def test_backward_mixed_dims_gqa(Dk, Dv, algo):
    """Dk != Dv with 3 value heads per query/key head (dq, dk summed over each
    group), bf16 inputs, chunk boundaries inside both sequences."""
    inp = inputs.prefill_inputs([150, 64], 1, 3, Dk, dtype="bf16", seed=151, init_std=0.1)
    gen = torch.Generator().manual_seed(152)
    T = 214
    v = torch.randn(T, 3, Dv, generator=gen).to(torch.bfloat16)
    s0 = torch.randn(2, 3, Dv, Dk, generator=gen) * 0.1
    d_o = torch.randn(T, 3, Dv, generator=gen)
    d_sf = torch.randn(2, 3, Dv, Dk, generator=gen) * 0.1
    out = api.prefill_backward(inp["q"].to(DEV), inp["k"].to(DEV), v.to(DEV), inp["g"].to(DEV),
                               inp["beta"].to(DEV), d_o.to(DEV), cu_seqlens=inp["cu_seqlens"].to(DEV),
                               initial_state=s0.to(DEV), d_final_state=d_sf.to(DEV), scale=0.7,
                               sequential=algo == "sequential")
    torch.cuda.synchronize()
    ref = oracle.backward(inp["q"], inp["k"], v, inp["g"], inp["beta"], d_o, cu_seqlens=inp["cu_seqlens"],
                          initial_state=s0, d_final_state=d_sf, scale=0.7)
    _check(out, ref, f"{algo} GQA Dk={Dk} Dv={Dv}")


def test_backward_without_states(algo):
    """No initial state and no final-state gradient (both NULL)."""
    out, ref = _case([70], 1, 3, 64, "fp32", seed=107, algo=algo, init=False, dsf=False, scale=1.0)
    _check(out, ref, f"{algo} no states")


def test_backward_long_sequence(algo):
    """1000 tokens (15 chunks of 64 plus a ragged one; 62 checkpoint intervals
    of 16 plus one for the sequential form) at D=64."""
    out, ref = _case([1000], 1, 2, 64, "bf16", seed=108, algo=algo)
    _check(out, ref, f"{algo} T=1000")


@pytest.mark.parametrize("Hqk,Hv,N", [(2, 6, 50), (2, 2, 150)])
def test_backward_many_units_one_slice(Hqk, Hv, N, algo):
    """Enough (sequence, value head) units to fill the GPU: one slice per head,
    dg and dbeta written directly (and dq, dk too when Hv == Hqk)."""
    lengths = [(7 * i) % 23 for i in range(N)]  # 0 .. 22 tokens, some empty
    out, ref = _case(lengths, Hqk, Hv, 64, "fp32", seed=109 + Hv, algo=algo)
    _check(out, ref, f"{algo} {N} sequences x {Hv} heads")


@pytest.mark.slow
def test_backward_prefill8k_all_heads():
    """The bench's backward workload at full size (8192 tokens, 16/48 heads,
    D=128, bf16 inputs) with an initial state and dL/dS_final, chunk form,
    every gradient element of every head against the oracle.  The oracle runs
    one query/key head (its 3 value heads) per call, calls in threads."""
    from concurrent.futures import ThreadPoolExecutor
    import os

    w = inputs.WORKLOADS["prefill8k"]
    inp = inputs.prefill_inputs(w.lengths, w.Hqk, w.Hv, w.D, dtype=w.dtype, seed=w.seed, init_std=0.02)
    T, G = sum(w.lengths), w.Hv // w.Hqk
    gen = torch.Generator().manual_seed(131)
    d_o = torch.randn(T, w.Hv, w.D, generator=gen)
    d_sf = torch.randn(1, w.Hv, w.D, w.D, generator=gen) * 0.1
    dev = {n: t.to(DEV) for n, t in inp.items() if t is not None}
    out = api.prefill_backward(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], d_o.to(DEV),
                               cu_seqlens=dev["cu_seqlens"], initial_state=dev["initial_state"],
                               d_final_state=d_sf.to(DEV))
    torch.cuda.synchronize()

    def ref(hk):
        qs, vs = slice(hk, hk + 1), slice(G * hk, G * hk + G)
        return hk, oracle.backward(inp["q"][:, qs], inp["k"][:, qs], inp["v"][:, vs], inp["g"][:, vs],
                                   inp["beta"][:, vs], d_o[:, vs], cu_seqlens=inp["cu_seqlens"],
                                   initial_state=inp["initial_state"][:, vs], d_final_state=d_sf[:, vs])

    workers = max(1, min(8, (os.cpu_count() or 1)))
    with ThreadPoolExecutor(workers) as ex:
        results = list(ex.map(ref, range(w.Hqk)))
    full = [np.zeros(tuple(t.shape)) for t in out]
    for hk, r in results:
        qs, vs = slice(hk, hk + 1), slice(G * hk, G * hk + G)
        full[0][:, qs], full[1][:, qs], full[2][:, vs] = r[0], r[1], r[2]
        full[3][:, vs], full[4][:, vs], full[5][:, vs] = r[3], r[4], r[5]
    _check(out, full, "prefill8k all heads")


@pytest.mark.slow
def test_backward_long_slow_decay():
    """16,384 tokens (256 chunks per head) with the long workload's slow decay
    (g = -softplus(N(-2, 1))) and an N(0, 0.02) initial state, one query/key
    head and its 3 value heads at D=128, bf16 inputs: both chains run 256
    chunks, so errors that grow along them would show; every gradient within
    1e-4 of RMS of the oracle, for both forms."""
    T = 16384
    inp = inputs.prefill_inputs([T], 1, 3, 128, dtype="bf16", seed=141, g_mu=-2.0, init_std=0.02)
    gen = torch.Generator().manual_seed(142)
    d_o = torch.randn(T, 3, 128, generator=gen)
    d_sf = torch.randn(1, 3, 128, 128, generator=gen) * 0.1
    dev = {n: t.to(DEV) for n, t in inp.items() if t is not None}
    ref = oracle.backward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], d_o,
                          cu_seqlens=inp["cu_seqlens"], initial_state=inp["initial_state"],
                          d_final_state=d_sf)
    for sequential in (False, True):
        out = api.prefill_backward(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], d_o.to(DEV),
                                   cu_seqlens=dev["cu_seqlens"], initial_state=dev["initial_state"],
                                   d_final_state=d_sf.to(DEV), sequential=sequential)
        torch.cuda.synchronize()
        _check(out, ref, f"{'sequential' if sequential else 'chunked'} T=16384 slow decay")
