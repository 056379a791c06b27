"""Checks that pin the fp64 oracle to what the definition fixes.

Each check builds its own small inputs, runs a given oracle build (the
in-tree library, or a mutated copy in the mutation tests) and raises
AssertionError when the oracle disagrees with a result fixed independently of
it: a hand-worked example, a closed form, an invariant of the rule, or a
brute-force evaluation of the explicit matrix-product form.

Definition ("Inside Qwen3.8-27B: Hybrid DeltaNet Architecture, 256k Context,
and 24GB Local Serving", section "Gated DeltaNet Mechanics"):
    S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = scale S_t q_t
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, rtol, what):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    scale = max(1.0, float(np.abs(b).max()) if b.size else 1.0)
    err = float(np.abs(a - b).max()) if a.size else 0.0
    assert err <= rtol * scale, f"{what}: max abs err {err:.3e} > {rtol:.1e} * {scale:.3e}"


def random_problem(seed, T, Hqk, Hv, Dk, Dv, normalise=True, init=True, N=1):
    r = _rng(seed)
    q = r.standard_normal((T, Hqk, Dk))
    k = r.standard_normal((T, Hqk, Dk))
    if normalise:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((T, Hv, Dv))
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((T, Hv))))
    g = -np.log1p(np.exp(r.standard_normal((T, Hv))))
    s0 = 0.3 * r.standard_normal((N, Hv, Dv, Dk)) if init else None
    return q, k, v, g, beta, s0


# --------------------------------------------------------------------------
# brute force: explicit matrix-product form, no shared code with the oracle
def product_form(S0, alpha, beta, k, v, q):
    """S_t = S0 A_1..A_t + sum_{s<=t} B_s A_{s+1}..A_t with
    A_t = alpha_t (I - beta_t k_t k_t^T), B_t = beta_t v_t k_t^T;
    returns (o [T, Dv] with o_t = S_t q_t, S_T)."""
    T, Dk = k.shape
    if T == 0:
        return np.zeros((0, S0.shape[0])), S0.copy()
    A = [alpha[t] * (np.eye(Dk) - beta[t] * np.outer(k[t], k[t])) for t in range(T)]
    B = [beta[t] * np.outer(v[t], k[t]) for t in range(T)]

    def chain(a, b):  # A_a @ ... @ A_b (0-based, inclusive); identity when a > b
        P = np.eye(Dk)
        for i in range(a, b + 1):
            P = P @ A[i]
        return P

    outs, S = [], S0.copy()
    for t in range(T):
        S = S0 @ chain(0, t)
        for s in range(t + 1):
            S = S + B[s] @ chain(s + 1, t)
        outs.append(S @ q[t])
    return np.array(outs).reshape(T, -1), S


def check_product_form(lib, seed=0, T=7, Hqk=1, Hv=2, Dk=4, Dv=3, scale=1.0):
    q, k, v, g, beta, s0 = random_problem(seed, T, Hqk, Hv, Dk, Dv, normalise=False)
    o, fin = oracle.prefill(q, k, v, g, beta, initial_state=s0, scale=scale, lib=lib)
    G = Hv // Hqk
    for h in range(Hv):
        j = h // G
        o_ref, S_ref = product_form(s0[0, h], np.exp(g[:, h]), beta[:, h], k[:, j], v[:, h], q[:, j])
        _close(o[:, h], scale * o_ref, 1e-12, f"o head {h}")
        _close(fin[0, h], S_ref, 1e-12, f"final state head {h}")


# --------------------------------------------------------------------------
# hand-worked examples
def check_golden_scalar(lib):
    with open(os.path.join(GOLDEN, "scalar_d1.json")) as f:
        gd = json.load(f)
    T = len(gd["alpha"])
    q = np.array(gd["q"]).reshape(T, 1, 1)
    k = np.array(gd["k"]).reshape(T, 1, 1)
    v = np.array(gd["v"]).reshape(T, 1, 1)
    g = np.log(np.array(gd["alpha"])).reshape(T, 1)
    beta = np.array(gd["beta"]).reshape(T, 1)
    s0 = np.array(gd["s0"]).reshape(1, 1, 1, 1)
    for split in range(T + 1):  # also through a resume at every split point
        if split in (0, T):
            o, fin = oracle.prefill(q, k, v, g, beta, initial_state=s0, lib=lib)
        else:
            o1, f1 = oracle.prefill(q[:split], k[:split], v[:split], g[:split], beta[:split],
                                    initial_state=s0, lib=lib)
            o2, fin = oracle.prefill(q[split:], k[split:], v[split:], g[split:], beta[split:],
                                     initial_state=f1, lib=lib)
            o = np.concatenate([o1, o2])
        _close(o.reshape(T), gd["o"], 1e-14, "scalar golden o")
        _close(fin.reshape(()), gd["s"][-1], 1e-14, "scalar golden state")


def check_golden_matrix(lib):
    with open(os.path.join(GOLDEN, "matrix_d2.json")) as f:
        gd = json.load(f)
    T = len(gd["alpha"])
    q = np.array(gd["q"]).reshape(T, 1, 2)
    k = np.array(gd["k"]).reshape(T, 1, 2)
    v = np.array(gd["v"]).reshape(T, 1, 2)
    g = np.log(np.array(gd["alpha"])).reshape(T, 1)
    beta = np.array(gd["beta"]).reshape(T, 1)
    s0 = np.array(gd["S0"]).reshape(1, 1, 2, 2)
    o, fin = oracle.prefill(q, k, v, g, beta, initial_state=s0, lib=lib)
    _close(o.reshape(T, 2), gd["o"], 1e-14, "matrix golden o")
    _close(fin.reshape(2, 2), gd["S"][-1], 1e-14, "matrix golden state")
    o1, f1 = oracle.prefill(q[:1], k[:1], v[:1], g[:1], beta[:1], initial_state=s0, lib=lib)
    _close(f1.reshape(2, 2), gd["S"][0], 1e-14, "matrix golden state after token 1")


# --------------------------------------------------------------------------
# invariants and closed forms
def check_no_write_no_decay(lib, seed=1):
    """beta = 0, alpha = 1: the state never changes and o_t = S0 q_t."""
    q, k, v, g, beta, s0 = random_problem(seed, 9, 2, 4, 5, 3)
    g[:] = 0.0
    beta[:] = 0.0
    o, fin = oracle.prefill(q, k, v, g, beta, initial_state=s0, lib=lib)
    _close(fin, s0, 1e-15, "state unchanged")
    for h in range(4):
        _close(o[:, h], q[:, h // 2] @ s0[0, h].T, 1e-14, "o = S0 q")


def check_exact_writeback(lib, seed=2):
    """alpha = 1, beta = 1, |k_t| = 1: after token t, S_t k_t = v_t exactly
    (the delta rule overwrites the value stored under k_t).  With q_t = k_t
    the output is therefore v_t."""
    q, k, v, g, beta, s0 = random_problem(seed, 11, 1, 3, 6, 4)
    g[:] = 0.0
    beta[:] = 1.0
    q = k.copy()
    o, _ = oracle.prefill(q, k, v, g, beta, initial_state=s0, lib=lib)
    _close(o, v, 1e-12, "S_t k_t = v_t")


def check_reset(lib, seed=3):
    """alpha = 0 (g = -inf): S_t = beta_t v_t k_t^T, o_t = beta_t (k_t.q_t) v_t."""
    q, k, v, g, beta, s0 = random_problem(seed, 6, 2, 6, 4, 5)
    g[:] = -np.inf
    o, fin = oracle.prefill(q, k, v, g, beta, initial_state=s0, lib=lib)
    for h in range(6):
        j = h // 3
        kq = np.sum(k[:, j] * q[:, j], axis=-1)
        _close(o[:, h], (beta[:, h] * kq)[:, None] * v[:, h], 1e-14, "o after reset")
        _close(fin[0, h], beta[-1, h] * np.outer(v[-1, h], k[-1, j]), 1e-14, "state after reset")


def check_pure_decay(lib, seed=4):
    """beta = 0: S_t = exp(g_1 + ... + g_t) S0 and o_t = exp(G_t) S0 q_t."""
    q, k, v, g, beta, s0 = random_problem(seed, 10, 1, 2, 3, 3)
    beta[:] = 0.0
    o, fin = oracle.prefill(q, k, v, g, beta, initial_state=s0, lib=lib)
    G = np.cumsum(g, axis=0)
    for h in range(2):
        _close(fin[0, h], math.exp(G[-1, h]) * s0[0, h], 1e-14, "decayed state")
        _close(o[:, h], np.exp(G[:, h])[:, None] * (q[:, 0] @ s0[0, h].T), 1e-14, "decayed o")


def check_orthonormal_memory(lib, D=4, T=13):
    """Keys e_{t mod D}, alpha = beta = 1, zero start: slot j holds the last
    value written to it, and querying e_j reads it back."""
    k = np.zeros((T, 1, D))
    q = np.zeros((T, 1, D))
    for t in range(T):
        k[t, 0, t % D] = 1.0
        q[t, 0, (3 * t + 1) % D] = 1.0
    v = _rng(5).standard_normal((T, 1, 2))
    g = np.zeros((T, 1))
    beta = np.ones((T, 1))
    o, fin = oracle.prefill(q, k, v, g, beta, lib=lib)
    last = {}
    for t in range(T):
        last[t % D] = v[t, 0]
        j = (3 * t + 1) % D
        _close(o[t, 0], last.get(j, np.zeros(2)), 1e-15, f"memory read t={t}")
    for j in range(D):
        _close(fin[0, 0][:, j], last.get(j, np.zeros(2)), 1e-15, f"slot {j}")


def check_scale(lib, seed=6):
    q, k, v, g, beta, s0 = random_problem(seed, 5, 1, 1, 3, 3)
    o1, f1 = oracle.prefill(q, k, v, g, beta, initial_state=s0, scale=1.0, lib=lib)
    o2, f2 = oracle.prefill(q, k, v, g, beta, initial_state=s0, scale=0.125, lib=lib)
    _close(o2, 0.125 * o1, 1e-15, "o scales with scale")
    _close(f2, f1, 0.0, "state does not depend on scale")


def check_gqa_mapping(lib, seed=7):
    """V head h reads query/key head h // (Hv / Hqk): each V head of a
    multi-head call equals a single-head call on that query/key head."""
    Hqk, Hv = 2, 6
    q, k, v, g, beta, s0 = random_problem(seed, 8, Hqk, Hv, 4, 4)
    o, fin = oracle.prefill(q, k, v, g, beta, initial_state=s0, lib=lib)
    for h in range(Hv):
        j = h // (Hv // Hqk)
        o1, f1 = oracle.prefill(q[:, j:j + 1], k[:, j:j + 1], v[:, h:h + 1], g[:, h:h + 1],
                                beta[:, h:h + 1], initial_state=s0[:, h:h + 1], lib=lib)
        _close(o[:, h], o1[:, 0], 0.0, f"head {h}")
        _close(fin[:, h], f1[:, 0], 0.0, f"head {h} state")


def check_varlen(lib, seed=8):
    """Packed sequences restart from their own initial state: a packed call
    equals separate calls (zero-length sequences included)."""
    lengths = [5, 0, 9, 1, 4]
    T = sum(lengths)
    q, k, v, g, beta, s0 = random_problem(seed, T, 1, 2, 3, 3, N=len(lengths))
    cu = np.concatenate([[0], np.cumsum(lengths)])
    o, fin = oracle.prefill(q, k, v, g, beta, cu_seqlens=cu, initial_state=s0, lib=lib)
    for n, L in enumerate(lengths):
        a, b = cu[n], cu[n + 1]
        o1, f1 = oracle.prefill(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b],
                                initial_state=s0[n:n + 1], lib=lib)
        _close(o[a:b], o1, 0.0, f"seq {n} o")
        _close(fin[n], f1[0], 0.0, f"seq {n} state")
        if L == 0:
            _close(fin[n], s0[n], 0.0, "empty sequence keeps its state")
    # each sequence also matches the brute-force product form
    for n in range(len(lengths)):
        a, b = cu[n], cu[n + 1]
        for h in range(2):
            o_ref, S_ref = product_form(s0[n, h], np.exp(g[a:b, h]), beta[a:b, h], k[a:b, 0],
                                        v[a:b, h], q[a:b, 0])
            if b > a:
                _close(o[a:b, h], o_ref, 1e-12, f"seq {n} head {h} product form")
            _close(fin[n, h], S_ref, 1e-12, f"seq {n} head {h} product state")


def check_decode(lib, seed=9):
    """One decode step per sequence equals the product form of one token."""
    B, Hqk, Hv, D = 3, 2, 4, 5
    r = _rng(seed)
    q = r.standard_normal((B, Hqk, D))
    k = r.standard_normal((B, Hqk, D))
    v = r.standard_normal((B, Hv, D))
    g = -np.log1p(np.exp(r.standard_normal((B, Hv))))
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((B, Hv))))
    S = r.standard_normal((B, Hv, D, D))
    o, S1 = oracle.decode_step(q, k, v, g, beta, S, lib=lib)
    for b in range(B):
        for h in range(Hv):
            j = h // 2
            o_ref, S_ref = product_form(S[b, h], np.exp(g[b, h:h + 1]), beta[b, h:h + 1],
                                        k[b, j:j + 1], v[b, h:h + 1], q[b, j:j + 1])
            _close(o[b, h], o_ref[0], 1e-13, "decode o")
            _close(S1[b, h], S_ref, 1e-13, "decode state")


def check_chunked(lib, seed=10):
    """The chunked WY/UT form reproduces the token-by-token recurrence for
    chunk sizes 1, 16 and 64 and lengths that are not a multiple of them."""
    lengths = [150, 64, 1, 70]
    T = sum(lengths)
    q, k, v, g, beta, s0 = random_problem(seed, T, 2, 6, 16, 8, N=len(lengths))
    cu = np.concatenate([[0], np.cumsum(lengths)])
    o_ref, f_ref = oracle.prefill(q, k, v, g, beta, cu_seqlens=cu, initial_state=s0, lib=lib)
    for C in (1, 16, 64):
        o, fin = oracle.prefill(q, k, v, g, beta, cu_seqlens=cu, initial_state=s0, chunk=C, lib=lib)
        _close(o, o_ref, 1e-11, f"chunked C={C} o")
        _close(fin, f_ref, 1e-11, f"chunked C={C} state")


def check_round_bf16(lib, seed=11):
    """bf16 at rest: round to nearest, ties to even, 8 significant bits.

    Hand-worked values of the format (the spacing of bf16 is 2^-7 in [1, 2),
    2^-133 below 2^-126, the largest finite value is (2 - 2^-7) 2^127), then
    torch's own fp32 -> bf16 conversion (an independent round-to-nearest-even)
    on random fp32 values and on constructed ties, where the fp64 -> bf16
    rounding of the oracle must agree exactly."""
    import torch

    cases = [
        (1 + 2 ** -8, 1.0),                       # tie between 1 and 1 + 2^-7: even is 1
        (1 + 3 * 2 ** -8, 1 + 2 ** -6),           # tie between 1 + 2^-7 and 1 + 2^-6: even is the upper
        (1 + 2 ** -8 + 2 ** -30, 1 + 2 ** -7),    # just above a tie
        (-(1 + 2 ** -8 + 2 ** -30), -(1 + 2 ** -7)),
        (1 + 2 ** -7 + 2 ** -9, 1 + 2 ** -7),     # below a tie
        (3 * 2 ** -9 + 2 ** -40, 3 * 2 ** -9),    # binade [2^-8, 2^-7), spacing 2^-15
        (0.5 * 2 ** -133, 0.0),                   # half the smallest subnormal: tie to even (zero)
        (0.75 * 2 ** -133, 2 ** -133),
        (3.2 * 2 ** -133, 3 * 2 ** -133),
        (255 * 2 ** 120 + 2 ** 119, math.inf),    # largest finite + half a spacing: tie, overflows
        (255 * 2 ** 120 + 2 ** 118, 255 * 2 ** 120),
        (0.0, 0.0), (-0.0, -0.0),
    ]
    got = oracle.round_bf16(np.array([c[0] for c in cases]), lib)
    for (x, want), y in zip(cases, got):
        assert y == want and math.copysign(1, y) == math.copysign(1, want), \
            f"round_bf16({x!r}) = {y!r}, want {want!r}"

    r = _rng(seed)
    f32 = (r.standard_normal(4096) * np.exp(r.uniform(-30, 30, 4096))).astype(np.float32)
    bits = r.integers(0, 2 ** 16, 512, dtype=np.uint32) << 16 | np.uint32(0x8000)  # exact ties
    bits = bits[(bits >> 23 & 0xFF) != 0xFF]                                  # finite ones
    f32 = np.concatenate([f32, bits.view(np.float32)])
    want = torch.from_numpy(f32).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_bf16(f32.astype(np.float64), lib)
    bad = np.flatnonzero(~((got == want) | (np.isnan(got) & np.isnan(want))))
    assert bad.size == 0, f"round_bf16 differs from fp32->bf16 RNE at {f32[bad[:3]]}: {got[bad[:3]]} vs {want[bad[:3]]}"


def check_state_at_rest_bf16(lib, seed=12):
    """With the state at rest in bf16, the returned final state is the exact
    fp64 one rounded once: every value is a bf16 value (it survives a round
    trip through torch.bfloat16 unchanged), lies within half a bf16 spacing of
    the exact value, and o is untouched by the rounding."""
    import torch

    q, k, v, g, beta, s0 = random_problem(seed, T=9, Hqk=1, Hv=2, Dk=8, Dv=4, N=2)
    cu = np.array([0, 4, 9])
    o_ex, f_ex = oracle.prefill(q, k, v, g, beta, cu, s0, lib=lib)
    o_r, f_r = oracle.prefill(q, k, v, g, beta, cu, s0, state_at_rest="bf16", lib=lib)
    assert np.array_equal(o_ex, o_r), "o must not depend on how the final state is stored"
    back = torch.from_numpy(f_r).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(back, f_r), "final state holds values that are not bf16"
    _, e = np.frexp(f_ex)
    half = np.ldexp(1.0, np.maximum(e - 9, -134))
    assert (np.abs(f_r - f_ex) <= half).all(), "rounded state is not the nearest bf16 value"
    assert not np.array_equal(f_r, f_ex), "rounding changed nothing: inputs too coarse to test it"


def check_prologue(lib, seed=13):
    """Input prologue (raw projections -> q, k, g, beta): hand-worked values and
    the identities that fix L2 normalisation, -softplus and sigmoid."""
    q = np.array([[[3.0, 4.0]], [[0.0, 0.0]]])
    k = np.array([[[1.0, 0.0]], [[0.0, -2.0]]])
    a = np.array([[0.0], [1.0]])
    b = np.array([[0.0], [math.log(3.0)]])
    qn, kn, g, beta = oracle.prologue(q, k, a, b, lib)
    _close(qn, [[[0.6, 0.8]], [[0.0, 0.0]]], 1e-15, "q normalised (zero row stays zero)")
    _close(kn, [[[1.0, 0.0]], [[0.0, -1.0]]], 1e-15, "k normalised")
    _close(g, [[-math.log(2.0)], [-math.log1p(math.e)]], 1e-15, "g = -softplus(a)")
    _close(beta, [[0.5], [0.75]], 1e-15, "beta = sigmoid(b)")

    r = _rng(seed)
    T, Hqk, Hv, D = 7, 2, 4, 16
    q = r.standard_normal((T, Hqk, D)) * 3.0
    k = r.standard_normal((T, Hqk, D)) * 0.1
    a = np.concatenate([r.standard_normal((T - 1, Hv)) * 4.0, [[50.0, -50.0, 0.0, 700.0]]])
    b = np.concatenate([r.standard_normal((T - 1, Hv)) * 4.0, [[50.0, -50.0, 0.0, -700.0]]])
    qn, kn, g, beta = oracle.prologue(q, k, a, b, lib)
    for x, xn, name in ((q, qn, "q"), (k, kn, "k")):
        _close(np.linalg.norm(xn, axis=-1), np.ones((T, Hqk)), 1e-14, f"|{name}^| = 1")
        _close((x * xn).sum(-1), np.linalg.norm(x, axis=-1), 1e-13, f"{name}^ along {name}")
    _close(np.exp(g), 1.0 / (1.0 + np.exp(np.minimum(a, 700.0))), 1e-15, "alpha = e^g = 1/(1+e^a)")
    _, _, g_neg, beta_neg = oracle.prologue(q, k, -a, -b, lib)
    _close(g_neg - g, a, 1e-12, "softplus(a) - softplus(-a) = a")
    _close(beta + beta_neg, np.ones_like(beta), 1e-15, "sigmoid(b) + sigmoid(-b) = 1")
    assert g[-1, 0] == -50.0 - math.log1p(math.exp(-50.0)) and g[-1, 3] == -700.0, "large a"
    assert 0.0 < beta[-1, 1] < 1e-21 and beta[-1, 0] == 1.0, "sigmoid tails"
    qn2, kn2, _, _ = oracle.prologue(qn, kn, a, b, lib)
    _close(qn2, qn, 1e-15, "normalising twice changes nothing")
    _close(kn2, kn, 1e-15, "normalising twice changes nothing (k)")


def check_backward_finite_differences(lib, seed=14, h=1e-6):
    """The backward pass against central finite differences of the forward
    definition: L = <dO, o> + <dS, S_final> over two packed sequences with GQA,
    initial states and a scale; every element of q, k, v, g, beta and the
    initial state is perturbed by +-h."""
    r = _rng(seed)
    cu = np.array([0, 2, 5])
    T, N, Hqk, Hv, Dk, Dv, scale = 5, 2, 1, 2, 3, 2, 0.7
    x = {"q": r.standard_normal((T, Hqk, Dk)), "k": 0.6 * r.standard_normal((T, Hqk, Dk)),
         "v": r.standard_normal((T, Hv, Dv)), "g": -np.abs(r.standard_normal((T, Hv))),
         "beta": r.uniform(0.1, 0.9, (T, Hv)), "s0": 0.5 * r.standard_normal((N, Hv, Dv, Dk))}
    dO = r.standard_normal((T, Hv, Dv))
    dS = r.standard_normal((N, Hv, Dv, Dk))

    def loss(a):
        o, f = oracle.prefill(a["q"], a["k"], a["v"], a["g"], a["beta"], cu_seqlens=cu,
                              initial_state=a["s0"], scale=scale, lib=lib)
        return float((o * dO).sum() + (f * dS).sum())

    grads = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], dO, cu_seqlens=cu,
                            initial_state=x["s0"], d_final_state=dS, scale=scale, lib=lib)
    for name, an in zip(("q", "k", "v", "g", "beta", "s0"), grads):
        num = np.zeros_like(x[name])
        for idx in np.ndindex(x[name].shape):
            a = {n: t.copy() for n, t in x.items()}
            a[name][idx] += h
            lp = loss(a)
            a[name][idx] -= 2 * h
            num[idx] = (lp - loss(a)) / (2 * h)
        _close(an, num, 1e-7, f"d{name} against finite differences")


ALL_CHECKS = [
    check_product_form, check_golden_scalar, check_golden_matrix, check_no_write_no_decay,
    check_exact_writeback, check_reset, check_pure_decay, check_orthonormal_memory, check_scale,
    check_gqa_mapping, check_varlen, check_decode, check_chunked, check_round_bf16,
    check_state_at_rest_bf16, check_prologue, check_backward_finite_differences,
]
