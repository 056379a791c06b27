"""fp64 CPU oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library and its Python
binding never import it, and it imports nothing from them.

The arithmetic lives in ``gdn_oracle.c`` (plain C, fp64, token by token);
this module compiles it with gcc, loads it with ctypes and converts inputs to
contiguous fp64 arrays.  bf16 and fp32 inputs convert to fp64 exactly, so the
oracle reads the very values the GPU reads.

Definition followed ("Inside Qwen3.8-27B: Hybrid DeltaNet Architecture, 256k
Context, and 24GB Local Serving", section "Gated DeltaNet Mechanics"):
    S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
    o_t = scale * S_t q_t,   alpha_t = exp(g_t).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

GCC_FLAGS = ["-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math", "-pthread"]


def build(src: str = _SRC, out: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile the oracle with gcc (IEEE fp64, no contraction) into ``out``."""
    cmd = ["gcc", *GCC_FLAGS, *extra_flags, "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _stale(lib_path: str, src: str) -> bool:
    return (not os.path.exists(lib_path)) or os.path.getmtime(lib_path) < os.path.getmtime(src)


def _bind(lib):
    d = ctypes.POINTER(ctypes.c_double)
    i64 = ctypes.POINTER(ctypes.c_int64)
    ci, cd = ctypes.c_int, ctypes.c_double
    lib.gdn_oracle_prefill.restype = ci
    lib.gdn_oracle_prefill.argtypes = [d, d, d, d, d, i64, ci, ci, ci, ci, ci, cd, d, d, d, ci, ci]
    lib.gdn_oracle_decode_step.restype = ci
    lib.gdn_oracle_decode_step.argtypes = [d, d, d, d, d, d, d, ci, ci, ci, ci, ci, cd, ci]
    lib.gdn_oracle_round_bf16.restype = ci
    lib.gdn_oracle_round_bf16.argtypes = [d, ctypes.c_int64]
    lib.gdn_oracle_prologue.restype = ci
    lib.gdn_oracle_prologue.argtypes = [d, d, d, d, ctypes.c_int64, ci, ci, ci]
    lib.gdn_oracle_backward.restype = ci
    lib.gdn_oracle_backward.argtypes = [d, d, d, d, d, i64, ci, ci, ci, ci, ci, cd, d, d, d,
                                        d, d, d, d, d, d]
    return lib


def load(lib_path: str | None = None):
    """Load (building first if needed) the oracle library.

    ``lib_path`` loads a specific build, e.g. a deliberately broken copy made
    by the mutation tests; the default is the in-tree ``liboracle.so``.
    """
    global _lib
    if lib_path is not None:
        return _bind(ctypes.CDLL(lib_path))
    with _lock:
        if _lib is None:
            if _stale(_LIB_PATH, _SRC):
                build()
            _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu")
        import torch

        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def round_bf16(x, lib=None):
    """x rounded to the nearest bf16 value (ties to even), in fp64: the value a
    state kept at rest in bf16 holds.  Returns a new fp64 array."""
    lib = lib or load()
    y = _f64(x).copy()
    rc = lib.gdn_oracle_round_bf16(_ptr(y), int(y.size))
    if rc != 0:
        raise ValueError(f"gdn_oracle_round_bf16 failed with code {rc}")
    return y


def prologue(q, k, a, b, lib=None):
    """Raw projections to the recurrence's inputs, in fp64: q, k [T, Hqk, Dk]
    L2-normalised per (token, head) row; g = -softplus(a) and beta = sigmoid(b)
    ([T, Hv]).  Leading dimensions may be any shape ([B, Tn, ...] for decode);
    returns new arrays (q, k, g, beta)."""
    lib = lib or load()
    q, k, g, beta = (_f64(t).copy() for t in (q, k, a, b))
    Dk, Hqk, Hv = q.shape[-1], q.shape[-2], g.shape[-1]
    T = q.size // (Dk * Hqk)
    assert k.shape == q.shape and beta.shape == g.shape and g.size == T * Hv
    rc = lib.gdn_oracle_prologue(_ptr(q), _ptr(k), _ptr(g), _ptr(beta), T, Hqk, Hv, Dk)
    if rc != 0:
        raise ValueError(f"gdn_oracle_prologue failed with code {rc}")
    return q, k, g, beta


def prefill(q, k, v, g, beta, cu_seqlens=None, initial_state=None, scale=1.0, chunk=0,
            num_threads=0, want_final=True, state_at_rest=None, lib=None):
    """Run the recurrence over packed sequences in fp64.

    q, k: [T, Hqk, Dk]; v: [T, Hv, Dv]; g, beta: [T, Hv]; cu_seqlens: [N+1]
    (default: one sequence of T tokens); initial_state: [N, Hv, Dv, Dk] or
    None (zeros).  chunk=0 is the token-by-token definition; chunk>0 the
    chunked WY/UT form.  state_at_rest="bf16" rounds the final state to bf16
    (a state stored in bf16 between calls; the arithmetic stays fp64).
    Returns (o [T, Hv, Dv], final_state [N, Hv, Dv, Dk]).
    """
    lib = lib or load()
    q, k, v, g, beta = (_f64(t) for t in (q, k, v, g, beta))
    T, Hqk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    assert k.shape == q.shape and v.shape[0] == T and g.shape == (T, Hv) and beta.shape == (T, Hv)
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    N = cu.shape[0] - 1
    s0 = _f64(initial_state)
    if s0 is not None:
        assert s0.shape == (N, Hv, Dv, Dk), s0.shape
    o = np.zeros((T, Hv, Dv), dtype=np.float64)
    fin = np.zeros((N, Hv, Dv, Dk), dtype=np.float64) if want_final else None
    rc = lib.gdn_oracle_prefill(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), N, Hqk, Hv, Dk, Dv, float(scale),
        _ptr(s0), _ptr(fin), _ptr(o), int(chunk), int(num_threads))
    if rc != 0:
        raise ValueError(f"gdn_oracle_prefill failed with code {rc}")
    if state_at_rest not in (None, "fp64", "bf16"):
        raise ValueError(f"unknown state_at_rest {state_at_rest!r}")
    if state_at_rest == "bf16" and fin is not None:
        fin = round_bf16(fin, lib)
    return o, fin


def decode_step(q, k, v, g, beta, state, scale=1.0, num_threads=0, state_at_rest=None, lib=None,
                in_place=False):
    """One token for each of B sequences.  q, k: [B, Hqk, Dk]; v: [B, Hv, Dv];
    g, beta: [B, Hv]; state: [B, Hv, Dv, Dk].  Returns (o [B, Hv, Dv],
    new_state) and leaves the argument ``state`` untouched, unless
    ``in_place`` is set: then ``state`` must be a C-contiguous fp64 array,
    which is updated and returned (no copy, for long runs over large
    batches); state_at_rest="bf16" rounds new_state to bf16."""
    lib = lib or load()
    q, k, v, g, beta = (_f64(t) for t in (q, k, v, g, beta))
    if in_place:
        if not (isinstance(state, np.ndarray) and state.dtype == np.float64
                and state.flags["C_CONTIGUOUS"]):
            raise ValueError("in_place needs a C-contiguous float64 state array")
        S = state
    else:
        S = _f64(state).copy()
    B, Hqk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    o = np.zeros((B, Hv, Dv), dtype=np.float64)
    rc = lib.gdn_oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S),
                                    _ptr(o), B, Hqk, Hv, Dk, Dv, float(scale), int(num_threads))
    if rc != 0:
        raise ValueError(f"gdn_oracle_decode_step failed with code {rc}")
    if state_at_rest not in (None, "fp64", "bf16"):
        raise ValueError(f"unknown state_at_rest {state_at_rest!r}")
    if state_at_rest == "bf16":
        if in_place:
            S[...] = round_bf16(S, lib)
        else:
            S = round_bf16(S, lib)
    return o, S


def backward(q, k, v, g, beta, d_o, cu_seqlens=None, initial_state=None, d_final_state=None,
             scale=1.0, lib=None):
    """Gradients of L = <d_o, o> + <d_final_state, S_final> with respect to q,
    k, v, g, beta and the initial state, in fp64, token by token (small inputs:
    every state of a sequence is kept).  Shapes as for prefill; d_o [T, Hv, Dv].
    Returns (dq, dk, dv, dg, dbeta, d_initial_state)."""
    lib = lib or load()
    q, k, v, g, beta, d_o = (_f64(t) for t in (q, k, v, g, beta, d_o))
    T, Hqk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    N = cu.shape[0] - 1
    s0, dsf = _f64(initial_state), _f64(d_final_state)
    dq = np.zeros_like(q); dk = np.zeros_like(k); dv = np.zeros_like(v)
    dg = np.zeros_like(g); db = np.zeros_like(beta)
    ds0 = np.zeros((N, Hv, Dv, Dk))
    rc = lib.gdn_oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                 cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), N, Hqk, Hv, Dk,
                                 Dv, float(scale), _ptr(s0), _ptr(d_o), _ptr(dsf), _ptr(dq), _ptr(dk),
                                 _ptr(dv), _ptr(dg), _ptr(db), _ptr(ds0))
    if rc != 0:
        raise ValueError(f"gdn_oracle_backward failed with code {rc}")
    return dq, dk, dv, dg, db, ds0
