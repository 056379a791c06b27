"""Multi-token decode over a slot pool (gdn_decode_tokens) on the GPU against
the fp64 oracle: each sequence's tokens are a prefill of that length from the
state in its source slot, and the result lands in its destination slot."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_recurrence_rule_b200 import api, inputs
from parity import assert_parity, state_error, state_error_bf16_rest, to_np

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _case(B, Tn, Hqk, Hv, D, dtype, seed, num_slots, pool_std=0.3):
    inp = inputs.prefill_inputs([Tn] * B, Hqk, Hv, D, dtype=dtype, seed=seed)
    gen = torch.Generator().manual_seed(seed + 1000)
    pool = torch.randn(num_slots, Hv, D, D, generator=gen) * pool_std
    x = {"q": inp["q"].view(B, Tn, Hqk, D), "k": inp["k"].view(B, Tn, Hqk, D),
         "v": inp["v"].view(B, Tn, Hv, D), "g": inp["g"].view(B, Tn, Hv),
         "beta": inp["beta"].view(B, Tn, Hv)}
    return inp, x, pool


def _oracle(inp, pool, src, scale=1.0, state_at_rest=None):
    init = pool[torch.tensor(src, dtype=torch.long)]
    return oracle.prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                          cu_seqlens=inp["cu_seqlens"], initial_state=init, scale=scale,
                          state_at_rest=state_at_rest)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Tn", [1, 3, 16])
def test_slots_against_oracle(dtype, D, Tn):
    B, Hqk, Hv, slots = 3, 2, 6, 7
    inp, x, pool = _case(B, Tn, Hqk, Hv, D, dtype, seed=31 + Tn, num_slots=slots)
    src, dst = [4, 0, 6], [2, 5, 1]
    pin = pool.to(DEV)
    pout = torch.full_like(pin, float("nan"))
    o = api.decode_tokens(*(x[n].to(DEV) for n in ("q", "k", "v", "g", "beta")), pin, pout,
                          src_slot=torch.tensor(src, dtype=torch.int32, device=DEV),
                          dst_slot=torch.tensor(dst, dtype=torch.int32, device=DEV), scale=0.5)
    torch.cuda.synchronize()
    o_ref, f_ref = _oracle(inp, pool, src, scale=0.5)
    o_gpu = to_np(o).reshape(B * Tn, Hv, D)
    assert_parity(inputs.DTYPES[dtype], o_gpu, o_ref, to_np(pout[dst]), f_ref, f"Tn={Tn}")
    untouched = [s for s in range(slots) if s not in dst]
    assert torch.isnan(pout[untouched]).all()          # only destination slots written
    assert torch.equal(pin.cpu(), pool)                 # the input pool is only read


def test_single_token_matches_decode_step():
    """tokens = 1 with the identity slot map is the decode step, bit for bit."""
    B, Hqk, Hv, D = 4, 2, 6, 128
    inp, x, pool = _case(B, 1, Hqk, Hv, D, "bf16", seed=40, num_slots=B)
    S1 = pool.to(DEV)
    S2 = pool.to(DEV)
    o1 = api.decode_tokens(*(x[n].to(DEV) for n in ("q", "k", "v", "g", "beta")), S1)
    o2 = api.decode_step(*(x[n][:, 0].to(DEV) for n in ("q", "k", "v", "g", "beta")), S2)
    torch.cuda.synchronize()
    assert torch.equal(o1[:, 0], o2) and torch.equal(S1, S2)


def test_in_place_padding_and_bad_slot():
    """In place (state_out = state_in); a padding entry (-1) reads and writes
    nothing; an out-of-range slot is reported and skipped."""
    B, Tn, Hqk, Hv, D, slots = 4, 4, 2, 6, 128, 5
    inp, x, pool = _case(B, Tn, Hqk, Hv, D, "bf16", seed=41, num_slots=slots)
    src = [3, -1, 9, 0]
    S = pool.to(DEV)
    o = torch.full((B, Tn, Hv, D), 7.0, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    api.decode_tokens(*(x[n].to(DEV) for n in ("q", "k", "v", "g", "beta")), S, o=o,
                      src_slot=torch.tensor(src, dtype=torch.int32, device=DEV),
                      device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == api.GDN_ERR_INVALID_ARG
    assert (o[1] == 7).all() and (o[2] == 7).all()      # padding and bad slot untouched
    for s in (1, 2, 4):
        assert torch.equal(S[s].cpu(), pool[s])          # slots nobody uses stay as they were
    keep = [0, 3]
    o_ref, f_ref = _oracle({n: (t.view(B, Tn, *t.shape[1:])[keep].reshape(-1, *t.shape[1:])
                                if n in ("q", "k", "v", "g", "beta") else t)
                            for n, t in inp.items() if n != "cu_seqlens"} |
                           {"cu_seqlens": torch.tensor([0, Tn, 2 * Tn], dtype=torch.int32)},
                           pool, [src[b] for b in keep])
    assert_parity(torch.bfloat16, to_np(o[keep]).reshape(-1, Hv, D), o_ref,
                  to_np(S[[src[b] for b in keep]]), f_ref, "in place")


# ---- states at rest in bf16 (fp32 arithmetic, one rounding per call) ---------

@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Tn", [1, 4, 16])
def test_bf16_state_against_oracle(dtype, D, Tn):
    """bf16 pool: the oracle reads the same bf16 values, runs the tokens in fp64
    and rounds the final state once; o within the input dtype's bound, the state
    within one rounding of the oracle's (and within the bf16 bound, 5e-3, of the
    unrounded result)."""
    B, Hqk, Hv, slots = 3, 2, 6, 7
    inp, x, pool = _case(B, Tn, Hqk, Hv, D, dtype, seed=51 + Tn, num_slots=slots)
    pool = pool.to(torch.bfloat16)
    src, dst = [4, 0, 6], [2, 5, 1]
    pin = pool.to(DEV)
    pout = torch.full_like(pin, float("nan"))
    o = api.decode_tokens(*(x[n].to(DEV) for n in ("q", "k", "v", "g", "beta")), pin, pout,
                          src_slot=torch.tensor(src, dtype=torch.int32, device=DEV),
                          dst_slot=torch.tensor(dst, dtype=torch.int32, device=DEV), scale=0.5)
    torch.cuda.synchronize()
    o_ref, f_ref = _oracle(inp, pool, src, scale=0.5, state_at_rest="bf16")
    _, f_exact = _oracle(inp, pool, src, scale=0.5)
    s_gpu = to_np(pout[dst])
    assert_parity(inputs.DTYPES[dtype], to_np(o).reshape(B * Tn, Hv, D), o_ref,
                  what=f"bf16 state Tn={Tn}")
    e = state_error_bf16_rest(s_gpu, f_ref)
    assert e <= 1.0, f"bf16 state Tn={Tn}: {e:.3f}x the one-rounding bound"
    # a state stored in bf16 is a bf16 quantity: the bf16 bound against the exact one
    assert state_error(s_gpu, f_exact) <= 5e-3
    untouched = [s for s in range(slots) if s not in dst]
    assert torch.isnan(pout[untouched].float()).all()
    assert torch.equal(pin.cpu(), pool)


@pytest.mark.parametrize("sdt", ["fp32", "bf16"])
@pytest.mark.parametrize("Tn", [1, 4])
def test_degenerate_gates(sdt, Tn):
    """alpha = 0 (g = -inf, the state resets), g = 0, beta = 0 and beta = 1 on
    chosen (sequence, token) pairs, against the oracle, on the fp32-pool and
    bf16-pool kernels."""
    B, Hqk, Hv, D, slots = 4, 2, 6, 128, 4
    inp, x, pool = _case(B, Tn, Hqk, Hv, D, "bf16", seed=81 + Tn, num_slots=slots)
    g, beta = inp["g"].view(B, Tn, Hv), inp["beta"].view(B, Tn, Hv)
    g[0, 0] = -float("inf")
    g[1, Tn - 1] = -float("inf")
    g[2] = 0.0
    beta[1, 0] = 0.0
    beta[2, Tn - 1] = 1.0
    beta[3] = 0.0
    if sdt == "bf16":
        pool = pool.to(torch.bfloat16)
    src = [0, 1, 2, 3]
    S = pool.to(DEV)
    o = api.decode_tokens(*(x[n].to(DEV) for n in ("q", "k", "v", "g", "beta")), S)
    torch.cuda.synchronize()
    o_gpu = to_np(o).reshape(B * Tn, Hv, D)
    assert np.isfinite(o_gpu).all() and torch.isfinite(S.float()).all()
    if sdt == "fp32":
        o_ref, f_ref = _oracle(inp, pool, src)
        assert_parity(torch.bfloat16, o_gpu, o_ref, to_np(S), f_ref, f"gates fp32 pool Tn={Tn}")
    else:
        o_ref, f_ref = _oracle(inp, pool, src, state_at_rest="bf16")
        _, f_exact = _oracle(inp, pool, src)
        assert_parity(torch.bfloat16, o_gpu, o_ref, what=f"gates bf16 pool Tn={Tn}")
        assert state_error_bf16_rest(to_np(S), f_ref) <= 1.0
        assert state_error(to_np(S), f_exact) <= 5e-3


def test_bf16_state_many_calls():
    """64 one-token calls and 16 four-token calls in place on a bf16 pool, each
    followed on the oracle by one rounding of the state: the two stay within the
    bf16-input bounds of each other (rounding flips of one bf16 spacing are the
    only source of divergence, and the recurrence damps them)."""
    B, Hqk, Hv, D = 4, 2, 6, 128
    for Tn, calls in ((1, 64), (4, 16)):
        inp, x, pool = _case(B, Tn * calls, Hqk, Hv, D, "bf16", seed=60 + Tn, num_slots=B)
        pool = pool.to(torch.bfloat16)
        S = pool.to(DEV)
        ref = pool.to(torch.float64).numpy()
        for c in range(calls):
            sl = slice(c * Tn, (c + 1) * Tn)
            xc = {n: x[n][:, sl].contiguous() for n in ("q", "k", "v", "g", "beta")}
            o = api.decode_tokens(*(xc[n].to(DEV) for n in ("q", "k", "v", "g", "beta")), S)
            o_ref, ref = oracle.prefill(
                *(xc[n].reshape(B * Tn, *xc[n].shape[2:]) for n in ("q", "k", "v", "g", "beta")),
                cu_seqlens=torch.arange(0, B * Tn + 1, Tn, dtype=torch.int32), initial_state=ref,
                state_at_rest="bf16")
        torch.cuda.synchronize()
        assert_parity(torch.bfloat16, to_np(o).reshape(B * Tn, Hv, D), o_ref, to_np(S), ref,
                      f"{calls} calls of {Tn}")
        assert state_error(to_np(S), ref) <= 1e-3, f"{calls} calls of {Tn}: state diverged"


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("in_place", [False, True])
def test_bf16_pool_many_units(D, in_place):
    """A batch large enough that the bf16-pool kernel's persistent CTAs take
    several (sequence, head) units each, double-buffering their states: a
    shuffled slot map, padding entries and an invalid slot mixed in, against
    the oracle (one rounding at rest) unit by unit."""
    B, Hqk, Hv, Tn = 300, 2, 6, 3
    slots = B + 20
    inp, x, pool = _case(B, Tn, Hqk, Hv, D, "bf16", seed=95 + D, num_slots=slots)
    pool = pool.to(torch.bfloat16)
    perm = torch.randperm(slots, generator=torch.Generator().manual_seed(7)).tolist()
    src = perm[:B]
    pad = set(range(5, B, 37))           # padding entries
    bad = 11                             # a real sequence with an invalid source slot
    src = [-1 if b in pad else s for b, s in enumerate(src)]
    src[bad] = slots + 3
    # destinations (out of place): distinct slots of another permutation
    dst = list(src) if in_place else perm[::-1][:B]
    pin = pool.to(DEV)
    pout = pin if in_place else torch.full_like(pin, float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = torch.full((B, Tn, Hv, D), 7.0, device=DEV)
    api.decode_tokens(*(x[n].to(DEV) for n in ("q", "k", "v", "g", "beta")), pin, pout,
                      src_slot=torch.tensor(src, dtype=torch.int32, device=DEV),
                      dst_slot=None if in_place else torch.tensor(dst, dtype=torch.int32, device=DEV),
                      o=o, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == api.GDN_ERR_INVALID_ARG      # the invalid slot, reported
    real = [b for b in range(B) if b not in pad and b != bad]
    for b in pad | {bad}:
        assert (o[b] == 7).all()                                # skipped: o untouched
    idx = torch.tensor(real)
    sub = inputs.prefill_inputs([Tn] * len(real), Hqk, Hv, D, dtype="bf16", seed=0)
    for n in ("q", "k", "v", "g", "beta"):
        sub[n] = x[n][idx].reshape(len(real) * Tn, *x[n].shape[2:]).contiguous()
    sub["cu_seqlens"] = torch.arange(0, len(real) * Tn + 1, Tn, dtype=torch.int32)
    o_ref, f_ref = _oracle(sub, pool, [src[b] for b in real], state_at_rest="bf16")
    assert_parity(torch.bfloat16, to_np(o[idx]).reshape(len(real) * Tn, Hv, D), o_ref,
                  what="many units")
    s_gpu = to_np(pout[torch.tensor([src[b] if in_place else dst[b] for b in real])])
    assert state_error_bf16_rest(s_gpu, f_ref) <= 1.0
