"""gdn_prefill_noalloc: the prefill entry point for callers that cannot
allocate device memory (their allocator belongs to a framework or runtime,
or the path cannot take cudaMalloc's device-wide synchronisation).  It keeps
its workspace in a static device array of the library.

Checked through the C ABI against the fp64 oracle, with the parity tolerances
of the prefill tests, on both of its paths (the single-pass tensor-core
kernel for bf16 at head dim 128, the CUDA-core kernel otherwise), on calls in
a row (the array is shared and must be cleared by each call), and that the
calls allocate no device memory.  This file is collected last on purpose; it
passes alone in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from gated_deltanet_recurrence_rule_b200 import api, inputs
import oracle
from parity import assert_parity, to_np

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _lib():
    lib = api.load()
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    lib.gdn_prefill_noalloc.restype = i32
    lib.gdn_prefill_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, i32,
                                        i32, f32, vp, vp, vp, vp, vp]
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(x, o, fin, status, scale=1.0):
    lib = _lib()
    T, Hqk, Dk = x["q"].shape
    Hv, Dv = x["v"].shape[1], x["v"].shape[2]
    N = x["cu_seqlens"].shape[0] - 1
    code = {torch.bfloat16: 0, torch.float32: 1}
    stream = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    return lib.gdn_prefill_noalloc(
        _ptr(x["q"]), _ptr(x["k"]), _ptr(x["v"]), _ptr(x["g"]), _ptr(x["beta"]),
        _ptr(x["cu_seqlens"]), N, T, Hqk, Hv, Dk, Dv, code[x["q"].dtype], code[o.dtype],
        float(scale), _ptr(x.get("initial_state")), _ptr(fin), _ptr(o), _ptr(status), stream)


def _case(seed, lengths, dtype="bf16", D=128):
    """(device inputs, CPU inputs) of a small packed case with initial states."""
    inp = inputs.prefill_inputs(lengths, 2, 6, D, dtype=dtype, seed=seed, init_std=0.05)
    return {n: t.to(DEV) for n, t in inp.items() if t is not None}, inp


def _outputs(x):
    T, Hv, Dv, Dk = x["q"].shape[0], x["v"].shape[1], x["v"].shape[2], x["q"].shape[2]
    N = x["cu_seqlens"].shape[0] - 1
    o = torch.full((T, Hv, Dv), float("nan"), device=DEV)
    fin = torch.full((N, Hv, Dv, Dk), float("nan"), device=DEV)
    status = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    return o, fin, status


def _check(case, status_expected=api.GDN_OK):
    x, cpu = case
    o, fin, status = _outputs(x)
    assert _noalloc(x, o, fin, status, scale=0.5) == api.GDN_OK
    torch.cuda.synchronize()
    assert int(status.item()) == status_expected
    o_ref, f_ref = oracle.prefill(cpu["q"], cpu["k"], cpu["v"], cpu["g"], cpu["beta"],
                                  cu_seqlens=cpu["cu_seqlens"], initial_state=cpu["initial_state"],
                                  scale=0.5)
    assert_parity(x["q"].dtype, to_np(o), o_ref, to_np(fin), f_ref, "noalloc")


def test_noalloc_matches_oracle_two_calls():
    _check(_case(31, [300]))                 # single-pass tensor-core kernel
    _check(_case(32, [1, 63, 65, 0, 130]))   # second call on the shared scratch


def test_noalloc_cuda_core_paths():
    _check(_case(35, [200, 0, 77], dtype="fp32"))          # fp32 inputs
    _check(_case(36, [129, 64, 3], dtype="bf16", D=64))    # bf16 at head dim 64


def test_noalloc_clears_status_between_calls():
    x, cpu = _case(33, [64, 64])
    bad = dict(x)
    bad["cu_seqlens"] = torch.tensor([0, 100, 90], dtype=torch.int32, device=DEV)
    o = torch.zeros((128, 6, 128), device=DEV)
    fin = torch.zeros((2, 6, 128, 128), device=DEV)
    status = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    assert _noalloc(bad, o, fin, status) == api.GDN_OK
    torch.cuda.synchronize()
    assert int(status.item()) == api.GDN_ERR_BAD_SEQLENS
    _check((x, cpu))                          # the next call starts from a cleared header
    _check(_case(34, [200], dtype="fp32"))    # CUDA-core path


def test_noalloc_allocates_nothing():
    """Warmed-up calls on both paths leave torch's allocator and the device's
    free memory exactly as they were."""
    cases = [_case(37, [300, 5]), _case(38, [100], dtype="fp32")]
    bufs = [_outputs(x) for x, _ in cases]
    for (x, _), (o, fin, status) in zip(cases, bufs):   # warm-up: module and kernel loading
        assert _noalloc(x, o, fin, status) == api.GDN_OK
    torch.cuda.synchronize()
    torch_before = torch.cuda.memory_allocated(DEV)
    free_before, _ = torch.cuda.mem_get_info(DEV)
    for _ in range(3):
        for (x, _), (o, fin, status) in zip(cases, bufs):
            assert _noalloc(x, o, fin, status) == api.GDN_OK
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated(DEV) == torch_before
    free_after, _ = torch.cuda.mem_get_info(DEV)
    assert free_after == free_before, f"device free memory changed by {free_before - free_after} B"
    for (o, fin, status) in bufs:
        assert int(status.item()) == api.GDN_OK
