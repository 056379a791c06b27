"""Thin ctypes binding over libgdn.so (C ABI declared in include/gdn.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libgdn.so.  PyTorch supplies device memory and the current CUDA
stream.  There is no CPU fallback: if the library is missing or the tensors
are not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_PKG, "libgdn.so")

GDN_OK = 0
GDN_ERR_INVALID_ARG = 1
GDN_ERR_UNSUPPORTED = 2
GDN_ERR_CUDA = 3
GDN_ERR_DEVICE_TIMEOUT = 4
GDN_ERR_BAD_SEQLENS = 5
GDN_ERR_WORKSPACE = 6
GDN_DTYPE_BF16 = 0
GDN_DTYPE_FP32 = 1
GDN_INPUT_PREPARED = 0
GDN_INPUT_RAW = 1

_DTYPE_CODE = {torch.bfloat16: GDN_DTYPE_BF16, torch.float32: GDN_DTYPE_FP32}

_lock = threading.Lock()
_lib = None


class GDNError(RuntimeError):
    """A libgdn call returned a nonzero status (or the library is missing)."""

    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status) if _lib else status}")


def load():
    """Load libgdn.so (raises GDNError if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(lib_path):
            raise GDNError(-1, f"libgdn.so is missing at {lib_path}; build it with "
                               "`python -m gated_deltanet_recurrence_rule_b200.build`")
        lib = ctypes.CDLL(lib_path)
        vp, i32, i64, sz, f32 = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                                 ctypes.c_float)
        lib.gdn_status_string.restype = ctypes.c_char_p
        lib.gdn_status_string.argtypes = [i32]
        lib.gdn_version.restype = i32
        lib.gdn_version.argtypes = []
        lib.gdn_prefill_workspace_size.restype = sz
        lib.gdn_prefill_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32, i32]
        lib.gdn_prefill_launch_count.restype = i64
        lib.gdn_prefill_launch_count.argtypes = [i32, i64, i32, i32, i32, i32, i32, sz]
        lib.gdn_prefill_workspace_size_rounds.restype = sz
        lib.gdn_prefill_workspace_size_rounds.argtypes = [i32, i64, i32, i32, i32, i32, i32, i64]
        lib.gdn_prefill.restype = i32
        lib.gdn_prefill.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, i32, i32,
                                    i32, i32, f32, vp, vp, vp, vp, sz, vp]
        lib.gdn_decode_step.restype = i32
        lib.gdn_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                        i32, f32, vp]
        lib.gdn_decode_tokens.restype = i32
        lib.gdn_decode_tokens.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, i32, i32, i32,
                                          i32, i32, i32, i32, i32, i32, i32, f32, vp, vp]
        lib.gdn_prefill_backward_workspace_size.restype = sz
        lib.gdn_prefill_backward_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32]
        lib.gdn_prefill_backward_workspace_size_sequential.restype = sz
        lib.gdn_prefill_backward_workspace_size_sequential.argtypes = [i32, i64, i32, i32, i32, i32]
        bwd_args = [vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, i32, f32, vp, vp, vp, vp,
                    vp, vp, vp, vp, vp, vp, sz, vp]
        for name in ("gdn_prefill_backward", "gdn_prefill_backward_sequential"):
            getattr(lib, name).restype = i32
            getattr(lib, name).argtypes = bwd_args
        lib.gdn_prefill_uses_tensor_cores.restype = i32
        lib.gdn_prefill_uses_tensor_cores.argtypes = [i32, i32, i32, i32, i32]
        lib.gdn_get_device_status.restype = i32
        lib.gdn_get_device_status.argtypes = [vp, vp, ctypes.POINTER(i32)]
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return load().gdn_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != GDN_OK:
        raise GDNError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _require(t, name, device, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def prefill_workspace_size(num_seqs, total_tokens, Hqk, Hv, Dk, Dv, dtype=torch.bfloat16,
                           chunks_per_round=0) -> int:
    """Workspace bytes for prefill; ``chunks_per_round`` > 0 bounds it by
    processing the packed chunk list in rounds of that many 64-token chunks."""
    lib = load()
    if chunks_per_round:
        return int(lib.gdn_prefill_workspace_size_rounds(num_seqs, total_tokens, Hqk, Hv, Dk, Dv,
                                                         _DTYPE_CODE[dtype], chunks_per_round))
    return int(lib.gdn_prefill_workspace_size(num_seqs, total_tokens, Hqk, Hv, Dk, Dv,
                                              _DTYPE_CODE[dtype]))


def prefill_launch_count(num_seqs, total_tokens, Hqk, Hv, Dk, Dv, workspace_bytes,
                         dtype=torch.bfloat16) -> int:
    """Kernel launches one prefill call makes with a workspace of that size."""
    return int(load().gdn_prefill_launch_count(num_seqs, total_tokens, Hqk, Hv, Dk, Dv,
                                               _DTYPE_CODE[dtype], workspace_bytes))


def prefill(q, k, v, g, beta, cu_seqlens=None, initial_state=None, output_final_state=True,
            final_state=None, scale=1.0, o=None, workspace=None, o_dtype=torch.float32,
            state_dtype=None, raw_inputs=False):
    """Chunked prefill over packed sequences on the GPU.

    q, k [T, Hqk, Dk]; v [T, Hv, Dv] (bf16 or fp32, same dtype); g, beta [T, Hv]
    fp32; cu_seqlens [N+1] int32 (default: one sequence of T tokens);
    o is produced in ``o_dtype`` (fp32 by default, or bf16);
    initial_state [N, Hv, Dv, Dk] or None (zeros).  ``final_state`` may
    be given (it may be ``initial_state`` itself, for an in-place update);
    otherwise one is allocated when ``output_final_state``.  States are fp32,
    or bf16 kept at rest (fp32 arithmetic, the final state rounded once): the
    dtype of the given states, else ``state_dtype`` (default fp32).
    ``raw_inputs``: q, k are raw projections (normalised in the kernels) and
    g, beta hold a, b with g = -softplus(a), beta = sigmoid(b).
    ``workspace``: a zero-filled uint8 CUDA tensor, reused across calls, or
    None (one of ``prefill_workspace_size`` bytes is allocated).  Its size
    selects the tensor-core schedule: full size runs the two phases; a
    256-byte one runs the single-pass kernel, which is faster for batches of
    many sequences of similar length and slower for a few long ones.
    Returns (o [T, Hv, Dv], final_state or None).
    """
    lib = load()
    if not q.is_cuda:
        raise ValueError("prefill runs on a CUDA device only (q is on the CPU)")
    dev = q.device
    T, Hqk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    dt = q.dtype
    if dt not in _DTYPE_CODE:
        raise ValueError(f"unsupported dtype {dt}")
    _require(q, "q", dev, dt)
    _require(k, "k", dev, dt, (T, Hqk, Dk))
    _require(v, "v", dev, dt, (T, Hv, Dv))
    _require(g, "g", dev, torch.float32, (T, Hv))
    _require(beta, "beta", dev, torch.float32, (T, Hv))
    if cu_seqlens is None:
        cu_seqlens = torch.tensor([0, T], dtype=torch.int32, device=dev)
    _require(cu_seqlens, "cu_seqlens", dev, torch.int32)
    N = cu_seqlens.shape[0] - 1
    sshape = (N, Hv, Dv, Dk)
    given = [t.dtype for t in (initial_state, final_state) if t is not None]
    sdt = given[0] if given else (state_dtype or torch.float32)
    if sdt not in _DTYPE_CODE or (state_dtype is not None and state_dtype != sdt):
        raise ValueError(f"unsupported or inconsistent state dtype {sdt}")
    if initial_state is not None:
        _require(initial_state, "initial_state", dev, sdt, sshape)
    if final_state is None and output_final_state:
        final_state = torch.empty(sshape, dtype=sdt, device=dev)
    if final_state is not None:
        _require(final_state, "final_state", dev, sdt, sshape)
    if o is None:
        o = torch.empty((T, Hv, Dv), dtype=o_dtype, device=dev)
    if o.dtype not in _DTYPE_CODE:
        raise ValueError(f"unsupported o dtype {o.dtype}")
    _require(o, "o", dev, None, (T, Hv, Dv))
    need = prefill_workspace_size(N, T, Hqk, Hv, Dk, Dv, dt)
    if workspace is None:
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    _require(workspace, "workspace", dev, torch.uint8)
    st = lib.gdn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), N, T,
                         Hqk, Hv, Dk, Dv, _DTYPE_CODE[dt], _DTYPE_CODE[o.dtype],
                         _DTYPE_CODE[sdt], GDN_INPUT_RAW if raw_inputs else GDN_INPUT_PREPARED,
                         float(scale), _ptr(initial_state),
                         _ptr(final_state), _ptr(o), _ptr(workspace), workspace.numel(),
                         _stream(dev))
    _check(st, "gdn_prefill")
    return o, final_state


def decode_step(q, k, v, g, beta, state, o=None, scale=1.0, o_dtype=torch.float32):
    """One token for each of B sequences; ``state`` [B, Hv, Dv, Dk] fp32 is
    updated in place.  q, k [B, Hqk, Dk]; v [B, Hv, Dv]; g, beta [B, Hv] fp32.
    Returns o [B, Hv, Dv] in ``o_dtype`` (fp32 by default, or bf16)."""
    lib = load()
    if not q.is_cuda:
        raise ValueError("decode_step runs on a CUDA device only (q is on the CPU)")
    dev = q.device
    B, Hqk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    dt = q.dtype
    if dt not in _DTYPE_CODE:
        raise ValueError(f"unsupported dtype {dt}")
    _require(q, "q", dev, dt)
    _require(k, "k", dev, dt, (B, Hqk, Dk))
    _require(v, "v", dev, dt, (B, Hv, Dv))
    _require(g, "g", dev, torch.float32, (B, Hv))
    _require(beta, "beta", dev, torch.float32, (B, Hv))
    _require(state, "state", dev, torch.float32, (B, Hv, Dv, Dk))
    if o is None:
        o = torch.empty((B, Hv, Dv), dtype=o_dtype, device=dev)
    if o.dtype not in _DTYPE_CODE:
        raise ValueError(f"unsupported o dtype {o.dtype}")
    _require(o, "o", dev, None, (B, Hv, Dv))
    st = lib.gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(o),
                             B, Hqk, Hv, Dk, Dv, _DTYPE_CODE[dt], _DTYPE_CODE[o.dtype],
                             float(scale), _stream(dev))
    _check(st, "gdn_decode_step")
    return o


def decode_tokens(q, k, v, g, beta, state_in, state_out=None, src_slot=None, dst_slot=None,
                  o=None, scale=1.0, o_dtype=torch.float32, device_status=None, raw_inputs=False):
    """Several tokens per sequence against a pool of states.

    q, k [B, Tn, Hqk, Dk]; v [B, Tn, Hv, Dv]; g, beta [B, Tn, Hv] fp32;
    state_in [num_slots, Hv, Dv, Dk] fp32 or bf16 (bf16: states at rest in
    bf16, fp32 arithmetic, rounded once per call on store); state_out the same
    shape and dtype (default: state_in, updated in place); src_slot / dst_slot
    [B] int32 or None (slot b / the source slot); device_status an int32 device
    tensor of one element or None.  ``raw_inputs`` as for prefill.  Returns o
    [B, Tn, Hv, Dv] in ``o_dtype``."""
    lib = load()
    if not q.is_cuda:
        raise ValueError("decode_tokens runs on a CUDA device only (q is on the CPU)")
    dev = q.device
    B, Tn, Hqk, Dk = q.shape
    Hv, Dv = v.shape[2], v.shape[3]
    dt = q.dtype
    if dt not in _DTYPE_CODE:
        raise ValueError(f"unsupported dtype {dt}")
    _require(q, "q", dev, dt)
    _require(k, "k", dev, dt, (B, Tn, Hqk, Dk))
    _require(v, "v", dev, dt, (B, Tn, Hv, Dv))
    _require(g, "g", dev, torch.float32, (B, Tn, Hv))
    _require(beta, "beta", dev, torch.float32, (B, Tn, Hv))
    num_slots = state_in.shape[0]
    sdt = state_in.dtype
    if sdt not in _DTYPE_CODE:
        raise ValueError(f"unsupported state dtype {sdt}")
    _require(state_in, "state_in", dev, sdt, (num_slots, Hv, Dv, Dk))
    if state_out is None:
        state_out = state_in
    _require(state_out, "state_out", dev, sdt, (num_slots, Hv, Dv, Dk))
    for name, sl in (("src_slot", src_slot), ("dst_slot", dst_slot)):
        if sl is not None:
            _require(sl, name, dev, torch.int32, (B,))
    if device_status is not None:
        _require(device_status, "device_status", dev, torch.int32, (1,))
    if o is None:
        o = torch.empty((B, Tn, Hv, Dv), dtype=o_dtype, device=dev)
    if o.dtype not in _DTYPE_CODE:
        raise ValueError(f"unsupported o dtype {o.dtype}")
    _require(o, "o", dev, None, (B, Tn, Hv, Dv))
    st = lib.gdn_decode_tokens(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in),
                               _ptr(state_out), _ptr(src_slot), _ptr(dst_slot), num_slots, _ptr(o),
                               B, Tn, Hqk, Hv, Dk, Dv, _DTYPE_CODE[dt], _DTYPE_CODE[o.dtype],
                               _DTYPE_CODE[sdt], GDN_INPUT_RAW if raw_inputs else GDN_INPUT_PREPARED,
                               float(scale), _ptr(device_status), _stream(dev))
    _check(st, "gdn_decode_tokens")
    return o


def prefill_backward(q, k, v, g, beta, d_o, cu_seqlens=None, initial_state=None,
                     d_final_state=None, scale=1.0, workspace=None, want_d_initial_state=True,
                     sequential=False):
    """Gradients of the prefill (fp32 states, prepared inputs) given d_o
    [T, Hv, Dv] fp32 and optionally d_final_state [N, Hv, Dv, Dk] fp32.
    Returns (dq, dk, dv, dg, dbeta, d_initial_state or None), all fp32.
    ``sequential`` calls gdn_prefill_backward_sequential (token by token);
    otherwise gdn_prefill_backward, which runs the chunk form when the
    workspace is large enough (the default one is)."""
    lib = load()
    if not q.is_cuda:
        raise ValueError("prefill_backward runs on a CUDA device only (q is on the CPU)")
    dev = q.device
    T, Hqk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    dt = q.dtype
    if dt not in _DTYPE_CODE:
        raise ValueError(f"unsupported dtype {dt}")
    _require(q, "q", dev, dt)
    _require(k, "k", dev, dt, (T, Hqk, Dk))
    _require(v, "v", dev, dt, (T, Hv, Dv))
    _require(g, "g", dev, torch.float32, (T, Hv))
    _require(beta, "beta", dev, torch.float32, (T, Hv))
    _require(d_o, "d_o", dev, torch.float32, (T, Hv, Dv))
    if cu_seqlens is None:
        cu_seqlens = torch.tensor([0, T], dtype=torch.int32, device=dev)
    _require(cu_seqlens, "cu_seqlens", dev, torch.int32)
    N = cu_seqlens.shape[0] - 1
    sshape = (N, Hv, Dv, Dk)
    for name, t in (("initial_state", initial_state), ("d_final_state", d_final_state)):
        if t is not None:
            _require(t, name, dev, torch.float32, sshape)
    f32 = dict(dtype=torch.float32, device=dev)
    dq, dk = torch.empty((T, Hqk, Dk), **f32), torch.empty((T, Hqk, Dk), **f32)
    dv = torch.empty((T, Hv, Dv), **f32)
    dg, db = torch.empty((T, Hv), **f32), torch.empty((T, Hv), **f32)
    ds0 = torch.empty(sshape, **f32) if want_d_initial_state else None
    size_fn = (lib.gdn_prefill_backward_workspace_size_sequential if sequential
               else lib.gdn_prefill_backward_workspace_size)
    need = size_fn(N, T, Hqk, Hv, Dk, Dv)
    if workspace is None:
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    _require(workspace, "workspace", dev, torch.uint8)
    fn = lib.gdn_prefill_backward_sequential if sequential else lib.gdn_prefill_backward
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens),
                                  N, T, Hqk, Hv, Dk, Dv, _DTYPE_CODE[dt], float(scale),
                                  _ptr(initial_state), _ptr(d_o), _ptr(d_final_state), _ptr(dq),
                                  _ptr(dk), _ptr(dv), _ptr(dg), _ptr(db), _ptr(ds0),
                                  _ptr(workspace), workspace.numel(), _stream(dev))
    _check(st, "gdn_prefill_backward_sequential" if sequential else "gdn_prefill_backward")
    return dq, dk, dv, dg, db, ds0


def prefill_backward_workspace_size(N, T, Hqk, Hv, Dk, Dv, sequential=False) -> int:
    """Workspace bytes gdn_prefill_backward needs for the chunk form, or with
    ``sequential`` the token-by-token form (0 for invalid sizes)."""
    lib = load()
    fn = (lib.gdn_prefill_backward_workspace_size_sequential if sequential
          else lib.gdn_prefill_backward_workspace_size)
    return int(fn(N, T, Hqk, Hv, Dk, Dv))


def prefill_uses_tensor_cores(Hqk, Hv, Dk, Dv, dtype=torch.bfloat16) -> bool:
    """Whether prefill with these sizes runs the tcgen05 tensor-core kernel."""
    return bool(load().gdn_prefill_uses_tensor_cores(Hqk, Hv, Dk, Dv, _DTYPE_CODE[dtype]))


def get_device_status(workspace) -> int:
    """Synchronise the current stream, return the sticky status word the
    prefills that used ``workspace`` left (GDN_OK or the first device-detected
    error code) and clear it."""
    lib = load()
    out = ctypes.c_int32(-1)
    st = lib.gdn_get_device_status(_ptr(workspace), _stream(workspace.device), ctypes.byref(out))
    _check(st, "gdn_get_device_status")
    return int(out.value)
