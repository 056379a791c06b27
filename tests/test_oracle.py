"""The fp64 oracle against what the definition fixes (CPU only).

See tests/oracle_pins.py for what each check pins and why it is independent
of the oracle's own code.
"""
import numpy as np
import pytest

import oracle
import oracle_pins as P


@pytest.mark.parametrize("D", [1, 2, 4, 8])
@pytest.mark.parametrize("T", [1, 5, 12])
def test_product_form(oracle_lib, D, T):
    P.check_product_form(oracle_lib, seed=D * 31 + T, T=T, Dk=D, Dv=max(1, D - 1))


def test_product_form_gqa_and_scale(oracle_lib):
    P.check_product_form(oracle_lib, seed=99, T=6, Hqk=2, Hv=6, Dk=3, Dv=2, scale=0.37)


@pytest.mark.parametrize("name", [c.__name__ for c in P.ALL_CHECKS if c is not P.check_product_form])
def test_pin(oracle_lib, name):
    getattr(P, name)(oracle_lib)


def test_thread_count_does_not_change_bits(oracle_lib):
    q, k, v, g, beta, s0 = P.random_problem(11, 40, 2, 6, 8, 8, N=2)
    cu = np.array([0, 17, 40])
    a = oracle.prefill(q, k, v, g, beta, cu_seqlens=cu, initial_state=s0, num_threads=1)
    b = oracle.prefill(q, k, v, g, beta, cu_seqlens=cu, initial_state=s0, num_threads=8)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_rejects_bad_cu_seqlens(oracle_lib):
    q, k, v, g, beta, s0 = P.random_problem(12, 6, 1, 1, 2, 2, init=False)
    with pytest.raises(ValueError):
        oracle.prefill(q, k, v, g, beta, cu_seqlens=np.array([0, 4, 3, 6]))
    with pytest.raises(ValueError):
        oracle.prefill(q, k, v, g, beta, cu_seqlens=np.array([1, 6]))


def test_empty_input(oracle_lib):
    q, k, v, g, beta, s0 = P.random_problem(13, 0, 1, 3, 2, 2)
    o, fin = oracle.prefill(q, k, v, g, beta, initial_state=s0)
    assert o.shape == (0, 3, 2)
    assert np.array_equal(fin, s0)


def test_bf16_state_drift_is_bounded(oracle_lib):
    """Tolerance study for states kept at rest in bf16 (oracle only): one token
    per call, the state rounded to bf16 after every call, against an fp64
    state kept throughout.  Each rounding adds relative noise of about 2^-9 and
    the recurrence damps old noise by alpha per step, so the error settles at
    about 2^-9 / sqrt(1 - alpha^2) instead of growing with the number of steps."""
    r = np.random.default_rng(5)
    B, Hv, D, steps, mu = 2, 3, 64, 256, -2.0
    S = oracle.round_bf16(0.02 * r.standard_normal((B, Hv, D, D)))
    exact, rest = S.copy(), S.copy()
    err = {}
    alphas = []
    for t in range(1, steps + 1):
        q = r.standard_normal((B, 1, D)); q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k = r.standard_normal((B, 1, D)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
        v = r.standard_normal((B, Hv, D))
        beta = 1 / (1 + np.exp(-r.standard_normal((B, Hv))))
        g = -np.log1p(np.exp(r.standard_normal((B, Hv)) + mu))
        alphas.append(np.exp(g))
        _, exact = oracle.decode_step(q, k, v, g, beta, exact, lib=oracle_lib)
        _, rest = oracle.decode_step(q, k, v, g, beta, rest, state_at_rest="bf16", lib=oracle_lib)
        if t in (64, 256):
            err[t] = np.linalg.norm(rest - exact) / np.linalg.norm(exact)
    a = float(np.median(np.concatenate(alphas, axis=None)))
    level = 2.0 ** -9 / np.sqrt(1 - a * a)
    assert 2.0 ** -11 < err[256] < 3 * level, (err, level)   # rounding happens, noise is damped
    assert err[256] < 2 * err[64], err                       # no growth with the number of steps


def test_decode_step_in_place_matches_copy(oracle_lib):
    """The wrapper's in-place mode only avoids the copy: same bits as the
    copying mode over several steps, with and without bf16 rounding at rest."""
    r = np.random.default_rng(21)
    B, Hqk, Hv, D = 3, 2, 6, 8
    for rest in (None, "bf16"):
        S_copy = r.standard_normal((B, Hv, D, D)) * 0.1
        S_in = S_copy.copy()
        for _ in range(4):
            q, k = r.standard_normal((B, Hqk, D)), r.standard_normal((B, Hqk, D))
            v = r.standard_normal((B, Hv, D))
            g, beta = -r.random((B, Hv)), r.random((B, Hv))
            o1, S_copy = oracle.decode_step(q, k, v, g, beta, S_copy, state_at_rest=rest)
            o2, S_ret = oracle.decode_step(q, k, v, g, beta, S_in, state_at_rest=rest, in_place=True)
            assert S_ret is S_in
            assert np.array_equal(o1, o2) and np.array_equal(S_copy, S_in)
    with pytest.raises(ValueError):
        oracle.decode_step(q, k, v, g, beta, S_in.astype(np.float32), in_place=True)
