"""The chunk form's reverse mode, written out in fp64, against the oracle (CPU only).

gdn_prefill_backward differentiates the chunked WY/UT form chunk by chunk
instead of token by token.  This module states those equations in plain numpy
(fp64, no blocking beyond the chunks themselves) and checks that they give the
oracle's token-by-token gradients, which finite differences pin in
oracle_pins.  So the algebra the CUDA kernels follow is pinned here on the CPU,
apart from their arithmetic, which the GPU tests compare with the oracle
element by element.

Chunk form ("Inside Qwen3.8-27B: Hybrid DeltaNet Architecture, 256k Context,
and 24GB Local Serving", section "Gated DeltaNet Mechanics").  Per chunk, with
G_t the running sum of the log-decays g, gamma_t = e^{G_t}, kdec_t =
e^{G_C - G_t} (C the chunk's last token) and E_ts = e^{G_t - G_s} for t >= s:
    A  = strict_lower(diag(beta) (E . K K^T)),   Tm = (I + A)^-1
    W  = Tm diag(beta gamma) K,   U~ = Tm diag(beta) V,   U = U~ - W S0^T
    O  = scale (diag(gamma) Q S0^T + (E . Q K^T) U)
    S1 = gamma_C S0 + U^T diag(kdec) K
The reverse mode below takes dO' = scale dO and dS1 (the gradient of the state
after the chunk) back through these products, last chunk first.
"""
import numpy as np
import pytest

import oracle


def _chunk_forward(Q, K, V, g, beta, S0, scale):
    """One chunk of one (sequence, value head): its outputs, the next state and
    the intermediates the reverse mode reads."""
    n = len(g)
    G = np.cumsum(g)
    gam, kdec = np.exp(G), np.exp(G[-1] - G)
    E = np.tril(np.exp(G[:, None] - G[None, :]))
    KK = K @ K.T
    A = np.tril(beta[:, None] * E * KK, -1)
    Tm = np.linalg.inv(np.eye(n) + A)
    W = Tm @ ((beta * gam)[:, None] * K)
    U = Tm @ (beta[:, None] * V) - W @ S0.T
    P = E * (Q @ K.T)
    O = scale * ((gam[:, None] * Q) @ S0.T + P @ U)
    S1 = gam[-1] * S0 + U.T @ (kdec[:, None] * K)
    return O, S1, dict(G=G, gam=gam, kdec=kdec, E=E, KK=KK, A=A, Tm=Tm, W=W, U=U, P=P)


def _chunk_reverse(Q, K, V, beta, S0, f, dO, dS1, scale):
    """Gradients of one chunk given dO (its outputs) and dS1 (the state after
    it).  Returns dq, dk, dv, dg, dbeta of its tokens and dS0."""
    gam, kdec, E, Tm, W, U, P = (f[x] for x in ("gam", "kdec", "E", "Tm", "W", "U", "P"))
    gC = gam[-1]
    dOp = scale * dO
    # the chain: dU, then the gradient of the state before the chunk
    dU = P.T @ dOp + kdec[:, None] * (K @ dS1.T)
    dS0 = gC * dS1 + dOp.T @ (gam[:, None] * Q) - dU.T @ W
    # O through P = E . Q K^T and diag(gamma) Q S0^T
    dP = np.tril(dOp @ U.T)
    dPE = dP * E
    dQ = gam[:, None] * (dOp @ S0) + dPE @ K
    dK = dPE.T @ Q + kdec[:, None] * (U @ dS1)
    dgam = np.sum(dOp * (Q @ S0.T), axis=1)
    dkdec = np.sum(U * (K @ dS1.T), axis=1)
    # U = Tm (diag(beta) V - diag(beta gamma) K S0^T) through Tm = (I + A)^-1
    dW = -dU @ S0
    dT = dW @ ((beta * gam)[:, None] * K).T + dU @ (beta[:, None] * V).T
    X, Y = Tm.T @ dW, Tm.T @ dU
    dK += (beta * gam)[:, None] * X
    dV = beta[:, None] * Y
    xk, yv = np.sum(X * K, axis=1), np.sum(Y * V, axis=1)
    dbeta = gam * xk + yv
    dgam += beta * xk
    dA = np.tril(-Tm.T @ dT @ Tm.T, -1)
    dbeta += np.sum(dA * E * f["KK"], axis=1)
    B = beta[:, None] * dA * E
    dK += (B + B.T) @ K
    # the decays: G enters through E (P and A), gamma, kdec and gamma_C
    dPP, dAA = dP * P, dA * f["A"]
    dG = dPP.sum(1) - dPP.sum(0) + dAA.sum(1) - dAA.sum(0) + dgam * gam - dkdec * kdec
    dG[-1] += np.sum(dkdec * kdec) + np.sum(dS1 * S0) * gC
    dg = np.cumsum(dG[::-1])[::-1]  # G_t sums g up to t
    return dQ, dK, dV, dg, dbeta, dS0


def _chunk_form(q, k, v, g, beta, dO, cu, s0, dSf, scale, C):
    """Forward outputs and gradients of every sequence and value head."""
    T, Hqk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    grp = Hv // Hqk
    o = np.zeros((T, Hv, Dv))
    fin = np.zeros((len(cu) - 1, Hv, Dv, Dk))
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dg, db = np.zeros_like(g), np.zeros_like(beta)
    ds0 = np.zeros_like(fin)
    for n in range(len(cu) - 1):
        a0, a1 = cu[n], cu[n + 1]
        for h in range(Hv):
            hk = h // grp
            S = s0[n, h].copy()
            saved = []
            for c0 in range(a0, a1, C):
                c1 = min(a1, c0 + C)
                O, S1, f = _chunk_forward(q[c0:c1, hk], k[c0:c1, hk], v[c0:c1, h], g[c0:c1, h],
                                          beta[c0:c1, h], S, scale)
                o[c0:c1, h] = O
                saved.append((c0, c1, S, f))
                S = S1
            fin[n, h] = S
            dS = dSf[n, h].copy()
            for c0, c1, S0, f in reversed(saved):
                r = _chunk_reverse(q[c0:c1, hk], k[c0:c1, hk], v[c0:c1, h], beta[c0:c1, h], S0, f,
                                   dO[c0:c1, h], dS, scale)
                dq[c0:c1, hk] += r[0]
                dk[c0:c1, hk] += r[1]
                dv[c0:c1, h], dg[c0:c1, h], db[c0:c1, h] = r[2], r[3], r[4]
                dS = r[5]
            ds0[n, h] = dS
    return (o, fin), (dq, dk, dv, dg, db, ds0)


def _problem(seed, lengths, Hqk, Hv, Dk, Dv):
    rng = np.random.default_rng(seed)
    T, N = sum(lengths), len(lengths)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q = unit(rng.standard_normal((T, Hqk, Dk)))
    k = unit(rng.standard_normal((T, Hqk, Dk)))
    v = rng.standard_normal((T, Hv, Dv))
    g = -np.log1p(np.exp(rng.standard_normal((T, Hv))))  # -softplus: alpha in (0, 1)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, Hv))))
    s0 = 0.3 * rng.standard_normal((N, Hv, Dv, Dk))
    dO = rng.standard_normal((T, Hv, Dv))
    dSf = rng.standard_normal((N, Hv, Dv, Dk))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return q, k, v, g, beta, s0, dO, dSf, cu


def _agree(got, want, what, tol=1e-9):
    for name, x, y in zip(what, got, want):
        rms = np.sqrt(np.mean(np.square(y))) if y.size else 0.0
        err = np.max(np.abs(x - y)) if y.size else 0.0
        assert err <= tol * max(rms, 1e-300), f"{name}: max error {err:.3e} against RMS {rms:.3e}"


CASES = {
    # lengths, Hqk, Hv, Dk, Dv, chunk
    "one_chunk_exact": ([64], 1, 1, 8, 8, 64),
    "ragged_tail": ([150], 1, 2, 6, 10, 64),
    "small_chunks_varlen": ([37, 0, 16, 5], 2, 6, 8, 12, 16),
    "gqa_three_value_heads": ([70, 33], 2, 6, 12, 8, 16),
}


@pytest.mark.parametrize("name", list(CASES))
def test_chunk_reverse_mode_matches_oracle(oracle_lib, name):
    lengths, Hqk, Hv, Dk, Dv, C = CASES[name]
    q, k, v, g, beta, s0, dO, dSf, cu = _problem(sum(lengths) + Hv, lengths, Hqk, Hv, Dk, Dv)
    scale = 0.6
    fwd, grads = _chunk_form(q, k, v, g, beta, dO, cu, s0, dSf, scale, C)
    _agree(fwd, oracle.prefill(q, k, v, g, beta, cu_seqlens=cu, initial_state=s0, scale=scale,
                               lib=oracle_lib), ["o", "final_state"])
    want = oracle.backward(q, k, v, g, beta, dO, cu_seqlens=cu, initial_state=s0, d_final_state=dSf,
                           scale=scale, lib=oracle_lib)
    _agree(grads, want, ["dq", "dk", "dv", "dg", "dbeta", "d_initial_state"])


def test_chunk_reverse_mode_degenerate_gates(oracle_lib):
    """alpha = 1 (g = 0), a strong decay (g = -20), beta = 0 and beta = 1 on
    chosen tokens, across chunk boundaries."""
    q, k, v, g, beta, s0, dO, dSf, cu = _problem(7, [45], 1, 3, 8, 8)
    g[[0, 15, 16, 31], :] = 0.0
    g[[5, 40], :] = -20.0
    beta[[3, 16, 44], :] = 0.0
    beta[[7, 17, 32], :] = 1.0
    fwd, grads = _chunk_form(q, k, v, g, beta, dO, cu, s0, dSf, 1.0, 16)
    _agree(fwd, oracle.prefill(q, k, v, g, beta, cu_seqlens=cu, initial_state=s0, lib=oracle_lib),
           ["o", "final_state"])
    want = oracle.backward(q, k, v, g, beta, dO, cu_seqlens=cu, initial_state=s0, d_final_state=dSf,
                           lib=oracle_lib)
    _agree(grads, want, ["dq", "dk", "dv", "dg", "dbeta", "d_initial_state"])
