"""The bounded-wait timeout path of the tensor-core prefill kernels, made to run
out on purpose without faulting or hanging anything.

Every mbarrier wait in the kernels gives up after the limit kept in the
workspace header (bytes 4-7, microseconds; 0 means the default of 2 s).
A limit of 1 us is shorter than any tile load, so some wait of the call runs
out: the kernel sets GDN_ERR_DEVICE_TIMEOUT in the status word, lets its own
copies and MMAs finish, frees its tensor memory and returns.  The test then
checks the status, and that the next ordinary call on the same GPU and the
same workspace still matches the oracle (the context stayed usable).
"""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_recurrence_rule_b200 import api, inputs
from parity import assert_parity, to_np

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")

WAIT_LIMIT_OFFSET = 4  # byte offset of the uint32 wait limit in the workspace header


def _set_wait_limit_us(ws, us):
    ws[WAIT_LIMIT_OFFSET:WAIT_LIMIT_OFFSET + 4].copy_(
        torch.tensor([us], dtype=torch.int32).view(torch.uint8).to(DEV))


def _workspace(path, N, T):
    if path == "two_phase":
        n = api.prefill_workspace_size(N, T, 2, 6, 128, 128)
    elif path == "rounds":
        n = api.prefill_workspace_size(N, T, 2, 6, 128, 128, chunks_per_round=3)
    else:  # single-pass kernel
        n = 256
    return torch.zeros(n, dtype=torch.uint8, device=DEV)


@pytest.mark.parametrize("path", ["two_phase", "rounds", "single_pass"])
def test_wait_limit_runs_out_then_next_call_is_correct(path):
    lengths = [1000, 300, 0, 77]
    inp = inputs.prefill_inputs(lengths, 2, 6, 128, dtype="bf16", seed=41, init_std=0.1)
    x = {n: t.to(DEV) for n, t in inp.items() if t is not None}
    N, T = len(lengths), sum(lengths)
    ws = _workspace(path, N, T)

    def call():
        return api.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], cu_seqlens=x["cu_seqlens"],
                           initial_state=x["initial_state"], workspace=ws)

    _set_wait_limit_us(ws, 1)
    call()
    assert api.get_device_status(ws) == api.GDN_ERR_DEVICE_TIMEOUT

    _set_wait_limit_us(ws, 0)
    o, f = call()
    assert api.get_device_status(ws) == api.GDN_OK
    o_ref, f_ref = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                  cu_seqlens=inp["cu_seqlens"], initial_state=inp["initial_state"])
    assert np.isfinite(to_np(o)).all()
    assert_parity(torch.bfloat16, to_np(o), o_ref, to_np(f), f_ref, f"after timeout, {path}")
