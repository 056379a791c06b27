"""Decode step on the GPU against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_recurrence_rule_b200 import api, inputs
from parity import TOL, assert_parity, o_error, state_error, to_np

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _step_inputs(d, s):
    return {n: d[n][s] for n in ("q", "k", "v", "g", "beta")}


@pytest.mark.parametrize("o_dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("Dk,Dv", [(64, 64), (128, 128), (128, 64), (64, 128)])
def test_decode_small(dtype, Dk, Dv, o_dtype):
    B, Hqk, Hv, steps = 3, 2, 6, 4
    d = inputs.decode_inputs(B, Hqk, Hv, Dk, steps=steps, dtype=dtype, seed=5, init_std=0.3, Dv=Dv)
    S_ref = d["state"].double().numpy()
    S = d["state"].to(DEV)
    for s in range(steps):
        x = _step_inputs(d, s)
        o = api.decode_step(*(x[n].to(DEV) for n in ("q", "k", "v", "g", "beta")), S, scale=0.5,
                            o_dtype=inputs.DTYPES[o_dtype])
        assert o.dtype == inputs.DTYPES[o_dtype]
        o_ref, S_ref = oracle.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], S_ref, scale=0.5)
        assert_parity(inputs.DTYPES[dtype], to_np(o), o_ref, to_np(S), S_ref, f"step {s}",
                      o_bf16=(o_dtype == "bf16"))


def test_decode_reset_and_no_write():
    """alpha = 0 (g = -inf) and beta = 0 edge cases."""
    B, Hqk, Hv, D = 2, 2, 6, 128
    d = inputs.decode_inputs(B, Hqk, Hv, D, steps=1, dtype="fp32", seed=6, init_std=0.3)
    x = _step_inputs(d, 0)
    x["g"][0] = -float("inf")
    x["beta"][1] = 0.0
    S = d["state"].to(DEV)
    o = api.decode_step(*(x[n].to(DEV) for n in ("q", "k", "v", "g", "beta")), S)
    o_ref, S_ref = oracle.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], d["state"])
    assert_parity(torch.float32, to_np(o), o_ref, to_np(S), S_ref, "reset")


def test_decode_guard_bands():
    """Nothing outside the state and output buffers is written."""
    B, Hqk, Hv, D = 4, 2, 6, 128
    d = inputs.decode_inputs(B, Hqk, Hv, D, steps=1, seed=7)
    n_state = B * Hv * D * D
    pad = 4096
    buf = torch.full((n_state + 2 * pad,), float("nan"), device=DEV)
    S = buf[pad:pad + n_state].view(B, Hv, D, D)
    S.copy_(d["state"].to(DEV))
    obuf = torch.full((B * Hv * D + 2 * pad,), 7.0, dtype=torch.bfloat16, device=DEV)
    o = obuf[pad:pad + B * Hv * D].view(B, Hv, D)
    x = _step_inputs(d, 0)
    api.decode_step(*(x[n].to(DEV) for n in ("q", "k", "v", "g", "beta")), S, o=o)
    torch.cuda.synchronize()
    assert torch.isnan(buf[:pad]).all() and torch.isnan(buf[-pad:]).all()
    assert (obuf[:pad] == 7).all() and (obuf[-pad:] == 7).all()
    assert not (o == 7).all()


def test_decode64_thousand_steps():
    """The batched decode workload (B=64, 16/48 heads, D=128, bf16, fp32
    state ~N(0, 0.02^2)) for 1000 consecutive steps, the whole batch tracked
    by the oracle: o of every (sequence, head) checked at every step, and the
    whole state after steps 1, 10, 100 and 1000."""
    w = inputs.WORKLOADS["decode64"]
    d = inputs.workload_inputs(w)
    S = d["state"].to(DEV)
    dev_in = {n: d[n].to(DEV) for n in ("q", "k", "v", "g", "beta")}
    S_ref = d["state"].double().numpy().copy()  # oracle state, updated in place
    to, ts = TOL[torch.bfloat16]
    worst_o = 0.0
    for s in range(w.steps):
        o = api.decode_step(dev_in["q"][s], dev_in["k"][s], dev_in["v"][s], dev_in["g"][s],
                            dev_in["beta"][s], S)
        o_ref, _ = oracle.decode_step(d["q"][s], d["k"][s], d["v"][s], d["g"][s], d["beta"][s],
                                      S_ref, in_place=True)
        worst_o = max(worst_o, o_error(to_np(o), o_ref))
        assert worst_o <= to, f"step {s + 1}: o error {worst_o:.3e}"
        if s + 1 in (1, 10, 100, 1000):
            es = state_error(to_np(S), S_ref)
            assert es <= ts, f"step {s + 1}: whole-batch state error {es:.3e}"
