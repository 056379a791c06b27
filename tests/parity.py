"""Shared parity helpers: run the fp64 oracle on the exact inputs the GPU
reads and compare with the tolerances of the gated delta rule workloads.

Tolerances (by input dtype; o produced in fp32):
  bf16 inputs, fp32 state:  max|o - o_ref| <= 1e-2 * RMS(o_ref)  and
                            ||S - S_ref||_F / ||S_ref||_F <= 5e-3
  fp32 inputs:              both bounds 1e-4
When o is stored in bf16, round-to-nearest-even adds at most 2^-8 |x| to
each element x, so the o bound becomes, element by element,
  |o - o_ref| <= tol * RMS(o_ref) * (1 + 2^-8) + 2^-8 |o_ref|.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL = {torch.bfloat16: (1e-2, 5e-3), torch.float32: (1e-4, 1e-4)}


def o_error(o, o_ref):
    o = np.asarray(o, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(o_ref ** 2))) if o_ref.size else 1.0
    err = float(np.abs(o - o_ref).max()) if o_ref.size else 0.0
    return err / max(rms, 1e-300)


def state_error(s, s_ref):
    s = np.asarray(s, dtype=np.float64)
    s_ref = np.asarray(s_ref, dtype=np.float64)
    den = float(np.linalg.norm(s_ref))
    num = float(np.linalg.norm(s - s_ref))
    if den == 0.0:
        return num
    return num / den


BF16_U = 2.0 ** -8  # unit roundoff of bf16 (8 significant bits)


def o_error_bf16(o, o_ref, tol):
    """Largest ratio of |o - o_ref| to the bf16-storage bound (<= 1 passes)."""
    o = np.asarray(o, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    if not o_ref.size:
        return 0.0
    rms = float(np.sqrt(np.mean(o_ref ** 2)))
    bound = tol * rms * (1 + BF16_U) + BF16_U * np.abs(o_ref)
    return float((np.abs(o - o_ref) / np.maximum(bound, 1e-300)).max())


def assert_parity(dtype, o, o_ref, s=None, s_ref=None, what="", o_bf16=False):
    to, ts = TOL[dtype]
    assert np.isfinite(np.asarray(o, dtype=np.float64)).all(), f"{what}: non-finite o"
    if o_bf16:
        eo = o_error_bf16(o, o_ref, to)
        assert eo <= 1.0, f"{what}: bf16 o exceeds its rounding-aware bound by {eo:.3f}x"
    else:
        eo = o_error(o, o_ref)
        assert eo <= to, f"{what}: max|o-o_ref|/RMS = {eo:.3e} > {to:.0e}"
    es = None
    if s is not None:
        es = state_error(s, s_ref)
        assert es <= ts, f"{what}: state rel Frobenius error {es:.3e} > {ts:.0e}"
    return eo, es


def state_error_bf16_rest(s, s_ref, slack_rel=2e-5):
    """Largest ratio of |s - s_ref| to the bound for states kept at rest in bf16
    (<= 1 passes).  s_ref is the oracle's state rounded once to bf16 (fp64
    arithmetic); s is the kernel's, computed in fp32 and rounded once.  With x
    the exact value and x' = x + e the fp32 one (|e| <= eps), the two roundings
    differ by at most half a bf16 spacing at each plus |e|, and a bf16 spacing
    at y is at most 2^-7 |y|, so
        |s - s_ref| <= 2^-7 (|s_ref| + 2 eps) + 2 eps,   eps = slack_rel * RMS(s_ref).
    """
    s = np.asarray(s, dtype=np.float64)
    s_ref = np.asarray(s_ref, dtype=np.float64)
    if not s_ref.size:
        return 0.0
    eps = slack_rel * float(np.sqrt(np.mean(s_ref ** 2)))
    bound = 2.0 ** -7 * (np.abs(s_ref) + 2 * eps) + 2 * eps
    return float((np.abs(s - s_ref) / np.maximum(bound, 1e-300)).max())


def to_np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def oracle_prefill_heads(inp, qk_heads, G, scale=1.0, num_threads=0):
    """Oracle on the subset of query/key heads ``qk_heads`` (and their G value
    heads each).  Returns (o [T, len*G, Dv], final [N, len*G, Dv, Dk], vheads)."""
    vheads = [j * G + r for j in qk_heads for r in range(G)]
    q = inp["q"][:, qk_heads]
    k = inp["k"][:, qk_heads]
    v = inp["v"][:, vheads]
    g = inp["g"][:, vheads]
    beta = inp["beta"][:, vheads]
    s0 = inp.get("initial_state")
    if s0 is not None:
        s0 = s0[:, vheads]
    o, fin = oracle.prefill(q, k, v, g, beta, cu_seqlens=inp["cu_seqlens"], initial_state=s0,
                            scale=scale, num_threads=num_threads)
    return o, fin, vheads
