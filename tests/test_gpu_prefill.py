"""Prefill on the GPU against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_recurrence_rule_b200 import api, inputs
from parity import TOL, assert_parity, oracle_prefill_heads, state_error, state_error_bf16_rest, to_np

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def run_gpu(inp, scale=1.0, alias=False, o_dtype=torch.float32):
    dev = {n: (t.to(DEV) if t is not None else None) for n, t in inp.items()}
    fin = dev["initial_state"] if alias else None
    o, f = api.prefill(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"],
                       cu_seqlens=dev["cu_seqlens"], initial_state=dev["initial_state"],
                       final_state=fin, scale=scale, o_dtype=o_dtype)
    torch.cuda.synchronize()
    return o, f


def run_oracle(inp, scale=1.0):
    return oracle.prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                          cu_seqlens=inp["cu_seqlens"], initial_state=inp["initial_state"],
                          scale=scale)


def test_tiny_workload():
    """T=256, Hqk=2, Hv=6, D=64, fp32, zero initial state, seed 0."""
    inp = inputs.workload_inputs(inputs.WORKLOADS["tiny"])
    o, f = run_gpu(inp)
    o_ref, f_ref = run_oracle(inp)
    assert_parity(torch.float32, to_np(o), o_ref, to_np(f), f_ref, "tiny")


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("D", [64, 128])
def test_ragged_chunks(dtype, D):
    """Several 64-token chunks plus a ragged tail, nonzero initial state."""
    inp = inputs.prefill_inputs([300], 2, 6, D, dtype=dtype, seed=11, init_std=0.1)
    o, f = run_gpu(inp, scale=0.75)
    o_ref, f_ref = run_oracle(inp, scale=0.75)
    assert_parity(inputs.DTYPES[dtype], to_np(o), o_ref, to_np(f), f_ref, f"{dtype} D={D}")


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_varlen_edges(dtype):
    """Packed sequences of length 1, 63, 64, 65, 0, 130 and 200 with their own
    initial states."""
    lengths = [1, 63, 64, 65, 0, 130, 200]
    inp = inputs.prefill_inputs(lengths, 2, 6, 128, dtype=dtype, seed=12, init_std=0.05)
    o, f = run_gpu(inp)
    o_ref, f_ref = run_oracle(inp)
    assert_parity(inputs.DTYPES[dtype], to_np(o), o_ref, to_np(f), f_ref, "varlen")
    # the empty sequence returns its initial state untouched
    assert torch.equal(f[4].cpu(), inp["initial_state"][4])


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_bf16_output(dtype):
    """o stored in bf16: checked against the rounding-aware bound."""
    inp = inputs.prefill_inputs([257, 64, 5], 2, 6, 128, dtype=dtype, seed=18, init_std=0.1)
    o, f = run_gpu(inp, o_dtype=torch.bfloat16)
    assert o.dtype == torch.bfloat16
    o_ref, f_ref = run_oracle(inp)
    assert_parity(inputs.DTYPES[dtype], to_np(o), o_ref, to_np(f), f_ref, "bf16 o", o_bf16=True)


def test_in_place_state():
    """final_state may be the initial_state buffer (updated in place)."""
    inp = inputs.prefill_inputs([129, 70], 2, 6, 128, dtype="bf16", seed=13, init_std=0.1)
    o, f = run_gpu(inp, alias=True)
    o_ref, f_ref = run_oracle(inp)
    assert_parity(torch.bfloat16, to_np(o), o_ref, to_np(f), f_ref, "aliased state")


def test_zero_tokens_copies_state():
    inp = inputs.prefill_inputs([0, 0], 2, 6, 64, dtype="bf16", seed=14, init_std=0.1)
    o, f = run_gpu(inp)
    assert o.shape[0] == 0
    assert torch.equal(f.cpu(), inp["initial_state"])


def test_reset_and_no_write_edges():
    """alpha = 0 on some tokens (state reset) and beta = 0 on others."""
    inp = inputs.prefill_inputs([200], 2, 6, 128, dtype="fp32", seed=15, init_std=0.1)
    inp["g"][[3, 64, 150]] = -float("inf")
    inp["beta"][[10, 11, 70]] = 0.0
    o, f = run_gpu(inp)
    o_ref, f_ref = run_oracle(inp)
    assert_parity(torch.float32, to_np(o), o_ref, to_np(f), f_ref, "edges")


@pytest.mark.parametrize("path", ["cuda_cores", "two_phase", "single_pass"])
def test_degenerate_gates(path):
    """alpha = 0 (g = -inf, the state resets) on single tokens, on the first and
    last token of a chunk and on a run of tokens; g = 0 (no decay) on a
    stretch; beta = 0 (no write) and beta = 1 (the key direction is replaced)
    on others; in both sequences of a packed batch, on every prefill path."""
    dtype = "fp32" if path == "cuda_cores" else "bf16"
    inp = inputs.prefill_inputs([260, 70], 2, 6, 128, dtype=dtype, seed=31, init_std=0.1)
    inp["g"][[3, 64, 127, 128, 129, 130, 200, 261]] = -float("inf")
    inp["g"][140:180] = 0.0
    inp["beta"][[10, 11, 70, 262]] = 0.0
    inp["beta"][[20, 90, 191, 300]] = 1.0
    if path == "single_pass":
        o, f = _run_ws(inp, torch.zeros(256, dtype=torch.uint8, device=DEV))
    else:
        o, f = run_gpu(inp)
    o_ref, f_ref = run_oracle(inp)
    assert np.isfinite(to_np(o)).all() and np.isfinite(to_np(f)).all()
    assert_parity(inputs.DTYPES[dtype], to_np(o), o_ref, to_np(f), f_ref, f"gates {path}")


def test_bad_cu_seqlens_sets_device_status():
    inp = inputs.prefill_inputs([64, 64], 2, 6, 64, dtype="bf16", seed=16)
    dev = {n: (t.to(DEV) if t is not None else None) for n, t in inp.items()}
    ws = torch.zeros(api.prefill_workspace_size(2, 128, 2, 6, 64, 64), dtype=torch.uint8, device=DEV)
    bad = torch.tensor([0, 100, 90], dtype=torch.int32, device=DEV)  # decreasing
    api.prefill(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], cu_seqlens=bad, workspace=ws)
    assert api.get_device_status(ws) == api.GDN_ERR_BAD_SEQLENS
    api.prefill(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], cu_seqlens=dev["cu_seqlens"],
                workspace=ws)
    assert api.get_device_status(ws) == api.GDN_OK


def test_guard_bands_and_determinism():
    inp = inputs.prefill_inputs([190, 3], 2, 6, 128, dtype="bf16", seed=17, init_std=0.1)
    dev = {n: (t.to(DEV) if t is not None else None) for n, t in inp.items()}
    T, pad = 193, 8192
    obuf = torch.full((T * 6 * 128 + 2 * pad,), 3.0, dtype=torch.bfloat16, device=DEV)
    o = obuf[pad:pad + T * 6 * 128].view(T, 6, 128)
    sbuf = torch.full((2 * 6 * 128 * 128 + 2 * pad,), float("nan"), device=DEV)
    f = sbuf[pad:pad + 2 * 6 * 128 * 128].view(2, 6, 128, 128)
    outs = []
    for _ in range(2):
        api.prefill(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"],
                    cu_seqlens=dev["cu_seqlens"], initial_state=dev["initial_state"],
                    final_state=f, o=o)
        torch.cuda.synchronize()
        outs.append((o.clone(), f.clone()))
    assert (obuf[:pad] == 3).all() and (obuf[-pad:] == 3).all()
    assert torch.isnan(sbuf[:pad]).all() and torch.isnan(sbuf[-pad:]).all()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def _run_ws(inp, ws):
    dev = {n: (t.to(DEV) if t is not None else None) for n, t in inp.items()}
    o, f = api.prefill(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"],
                       cu_seqlens=dev["cu_seqlens"], initial_state=dev["initial_state"],
                       workspace=ws)
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == api.GDN_OK
    return o, f


@pytest.mark.parametrize("rc", [1, 3, 7])
def test_rounds_bounded_workspace(rc):
    """A workspace for rounds of rc chunks: sequences cross round boundaries
    (state carried through the workspace); same bits as one round, and the
    oracle's result within tolerance."""
    lengths = [300, 1, 0, 130, 700, 64, 65]
    inp = inputs.prefill_inputs(lengths, 2, 6, 128, dtype="bf16", seed=19, init_std=0.1)
    N, T = len(lengths), sum(lengths)
    full = api.prefill_workspace_size(N, T, 2, 6, 128, 128)
    small = api.prefill_workspace_size(N, T, 2, 6, 128, 128, chunks_per_round=rc)
    assert small < full
    o1, f1 = _run_ws(inp, torch.zeros(full, dtype=torch.uint8, device=DEV))
    o2, f2 = _run_ws(inp, torch.zeros(small, dtype=torch.uint8, device=DEV))
    assert torch.equal(o1, o2) and torch.equal(f1, f2)
    o_ref, f_ref = run_oracle(inp)
    assert_parity(torch.bfloat16, to_np(o2), o_ref, to_np(f2), f_ref, f"rounds of {rc}")


def test_single_pass_header_workspace():
    """A 256-byte workspace runs the single-pass tensor-core kernel."""
    inp = inputs.prefill_inputs([300, 0, 65], 2, 6, 128, dtype="bf16", seed=20, init_std=0.1)
    o, f = _run_ws(inp, torch.zeros(256, dtype=torch.uint8, device=DEV))
    o_ref, f_ref = run_oracle(inp)
    assert_parity(torch.bfloat16, to_np(o), o_ref, to_np(f), f_ref, "single pass")


def _full_workload(name, alias=False, group=4):
    """The GPU prefill of a named workload against the oracle on EVERY head:
    the oracle runs on groups of ``group`` query/key heads (with their value
    heads) to bound host memory, and the errors are combined over the whole
    call: max |o - o_ref| over all outputs against RMS of all oracle outputs,
    and the relative Frobenius error of all final states."""
    w = inputs.WORKLOADS[name]
    inp = inputs.workload_inputs(w)
    o, f = run_gpu(inp, alias=alias)
    G = w.Hv // w.Hqk
    worst = sumsq = ds2 = s2 = 0.0
    count = 0
    for j0 in range(0, w.Hqk, group):
        heads = list(range(j0, min(j0 + group, w.Hqk)))
        o_ref, f_ref, vh = oracle_prefill_heads(inp, heads, G)
        og = to_np(o[:, vh])
        np.subtract(og, o_ref, out=og)
        np.abs(og, out=og)
        worst = max(worst, float(og.max()))
        del og
        sumsq += float(np.vdot(o_ref.ravel(), o_ref.ravel()))
        count += o_ref.size
        del o_ref
        fg = to_np(f[:, vh])
        ds2 += float(np.sum((fg - f_ref) ** 2))
        s2 += float(np.sum(f_ref ** 2))
    assert np.isfinite(worst)
    eo = worst / np.sqrt(sumsq / count)
    es = np.sqrt(ds2 / s2)
    to, ts = TOL[torch.bfloat16]
    assert eo <= to, f"{name}: max|o-o_ref|/RMS = {eo:.3e} > {to:.0e} (all {w.Hv} value heads)"
    assert es <= ts, f"{name}: state rel Frobenius error {es:.3e} > {ts:.0e}"
    return eo, es


def test_prefill8k_all_heads():
    """T=8192, 16/48 heads, D=128, bf16: every output and the final state of
    all 48 value heads against the oracle."""
    _full_workload("prefill8k", group=16)


@pytest.mark.slow
def test_long262k_all_heads_in_place():
    """T=262,144, slow decay, nonzero N(0,0.02) initial state returned as the
    final state in the same buffer (final_state == initial_state): all 48
    value heads against the oracle."""
    _full_workload("long262k", alias=True, group=4)


@pytest.mark.slow
def test_varlen32_all_heads():
    """32 packed sequences of 1024..32768 tokens with their own initial
    states: all 48 value heads of every sequence against the oracle."""
    _full_workload("varlen32", group=4)


# ---- states at rest in bf16: widened on load, rounded once on store ----------

def _bf16_state_case(lengths, dtype, D, seed, ws_bytes=None, alias=False):
    """Run the prefill with bf16 states, and again with fp32 states holding the
    same values; return both results and the oracle's."""
    inp = inputs.prefill_inputs(lengths, 2, 6, D, dtype=dtype, seed=seed, init_std=0.1)
    inp["initial_state"] = inp["initial_state"].to(torch.bfloat16)
    dev = {n: (t.to(DEV) if t is not None else None) for n, t in inp.items()}
    out = {}
    for sdt in (torch.bfloat16, torch.float32):
        ws = None if ws_bytes is None else torch.zeros(ws_bytes, dtype=torch.uint8, device=DEV)
        s0 = dev["initial_state"].to(sdt, copy=True)  # each run gets its own (in-place) copy
        o, f = api.prefill(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"],
                           cu_seqlens=dev["cu_seqlens"], initial_state=s0,
                           final_state=s0 if alias else None, workspace=ws)
        torch.cuda.synchronize()
        assert f.dtype == sdt
        if ws is not None:
            assert api.get_device_status(ws) == api.GDN_OK
        out[sdt] = (o, f)
    o_ref, f_ref = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                  cu_seqlens=inp["cu_seqlens"], initial_state=inp["initial_state"],
                                  state_at_rest="bf16")
    _, f_exact = run_oracle(inp)
    return inp, out, o_ref, f_ref, f_exact


def _check_bf16_states(inp, out, o_ref, f_ref, f_exact, dtype, slack_rel, what):
    """Exact against the same kernel with fp32 states (o bit for bit; the bf16
    final state is the fp32 one rounded to nearest even, bit for bit), and
    against the oracle: o within the input dtype's bound, the state within the
    bf16 bound of the exact one and within one rounding (plus the path's fp32
    error, slack_rel * RMS) of the oracle's rounded state."""
    o, f = out[torch.bfloat16]
    o32, f32 = out[torch.float32]
    assert torch.equal(o, o32), f"{what}: o depends on the state storage"
    assert torch.equal(f, f32.to(torch.bfloat16)), f"{what}: bf16 state is not RNE of the fp32 one"
    assert_parity(inputs.DTYPES[dtype], to_np(o), o_ref, what=what)
    e = state_error_bf16_rest(to_np(f), f_ref, slack_rel=slack_rel)
    assert e <= 1.0, f"{what}: {e:.3f}x the one-rounding bound"
    assert state_error(to_np(f), f_exact) <= 5e-3, what
    lengths = np.diff(inp["cu_seqlens"].numpy())
    for n in np.flatnonzero(lengths == 0):  # empty sequences: final state = initial state, bit for bit
        assert torch.equal(f[n].cpu(), inp["initial_state"][n]), f"{what}: empty sequence {n}"


# fp32 state error of the tensor-core path (bf16 operands with hi/lo splits),
# element by element, as a fraction of RMS(S)
TC_SLACK = 2e-3


@pytest.mark.parametrize("alias", [False, True])
def test_bf16_states_two_phase(alias):
    """Two-phase tensor-core prefill, full workspace, varlen with an empty
    sequence; bf16 initial and final states (also updated in place)."""
    lengths = [300, 0, 130, 64, 65]
    args = _bf16_state_case(lengths, "bf16", 128, seed=71, alias=alias)
    _check_bf16_states(*args, "bf16", TC_SLACK, f"two-phase alias={alias}")


def test_bf16_states_rounds_carry():
    """Rounds of 3 chunks: states cross rounds through the fp32 carry; only the
    caller's states are bf16."""
    lengths = [300, 1, 0, 130, 700, 64, 65]
    N, T = len(lengths), sum(lengths)
    ws = api.prefill_workspace_size(N, T, 2, 6, 128, 128, chunks_per_round=3)
    args = _bf16_state_case(lengths, "bf16", 128, seed=72, ws_bytes=ws)
    _check_bf16_states(*args, "bf16", TC_SLACK, "rounds of 3")


def test_bf16_states_single_pass():
    """Header-only workspace: the single-pass tensor-core kernel."""
    args = _bf16_state_case([300, 0, 65], "bf16", 128, seed=73, ws_bytes=256)
    _check_bf16_states(*args, "bf16", TC_SLACK, "single pass")


@pytest.mark.parametrize("D", [64, 128])
def test_bf16_states_cuda_cores(D):
    """fp32 inputs run the CUDA-core kernel; bf16 states there too."""
    args = _bf16_state_case([200, 0, 77], "fp32", D, seed=74 + D)
    _check_bf16_states(*args, "fp32", 2e-5, f"CUDA cores D={D}")


def test_bf16_states_zero_tokens():
    """T = 0: every sequence is empty and its bf16 final state is its initial state."""
    inp = inputs.prefill_inputs([0, 0], 2, 6, 128, dtype="bf16", seed=75, init_std=0.1)
    s0 = inp["initial_state"].to(torch.bfloat16).to(DEV)
    dev = {n: (t.to(DEV) if t is not None else None) for n, t in inp.items()}
    o, f = api.prefill(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"],
                       cu_seqlens=dev["cu_seqlens"], initial_state=s0)
    torch.cuda.synchronize()
    assert torch.equal(f, s0)


def test_two_caller_streams_own_workspaces():
    """Prefills issued on two caller streams, each with its own workspace and
    interleaved on the host: each stream gets its own internal stream pair,
    and both results match the oracle."""
    cases = [inputs.prefill_inputs([700, 129], 2, 6, 128, dtype="bf16", seed=81, init_std=0.1),
             inputs.prefill_inputs([300, 900, 5], 2, 6, 128, dtype="bf16", seed=82, init_std=0.1)]
    devs = [{n: t.to(DEV) for n, t in c.items() if t is not None} for c in cases]
    wss = [torch.zeros(api.prefill_workspace_size(x["cu_seqlens"].shape[0] - 1, x["q"].shape[0],
                                                  2, 6, 128, 128), dtype=torch.uint8, device=DEV)
           for x in devs]
    streams = [torch.cuda.Stream(DEV), torch.cuda.Stream(DEV)]
    torch.cuda.synchronize()
    outs = [None, None]
    for _ in range(3):
        for i, (x, ws, st) in enumerate(zip(devs, wss, streams)):
            with torch.cuda.stream(st):
                outs[i] = api.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"],
                                      cu_seqlens=x["cu_seqlens"], initial_state=x["initial_state"],
                                      workspace=ws)
    torch.cuda.synchronize()
    for c, ws, (o, f) in zip(cases, wss, outs):
        assert api.get_device_status(ws) == api.GDN_OK
        o_ref, f_ref = run_oracle(c)
        assert_parity(torch.bfloat16, to_np(o), o_ref, to_np(f), f_ref, "two caller streams")
