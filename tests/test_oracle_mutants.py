"""Plant plausible mistakes in a copy of the oracle and check the pins catch
every one of them (CPU only; the in-tree oracle is never modified).

Each mutant is a one-token textual edit of oracle/gdn_oracle.c compiled into
a temporary library.  A pin suite that still passed on one of them would not
be able to tell that mistake from the definition.
"""
import os

import pytest

import oracle
import oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")

# (name, text in the oracle, replacement)
MUTANTS = [
    ("erase_without_decay", "const double w = b * (vt[i] - alpha * u);",
     "const double w = b * (vt[i] - u);"),
    ("no_beta_on_write", "const double w = b * (vt[i] - alpha * u);",
     "const double w = (vt[i] - alpha * u);"),
    ("state_not_decayed", "Si[c] = alpha * Si[c] + w * kt[c];", "Si[c] = Si[c] + w * kt[c];"),
    ("write_with_query", "Si[c] = alpha * Si[c] + w * kt[c];", "Si[c] = alpha * Si[c] + w * qt[c];"),
    ("read_with_query", "u += Si[c] * kt[c];", "u += Si[c] * qt[c];"),
    ("output_with_key", "acc += Si[c] * qt[c];", "acc += Si[c] * kt[c];"),
    ("decay_sign", "const double alpha = exp(J->g[t * Hv + h]);",
     "const double alpha = exp(-J->g[t * Hv + h]);"),
    ("scale_dropped", "ot[i] = J->scale * acc;", "ot[i] = acc;"),
    ("gqa_modulo", "const int j = h / (Hv / Hqk); /* query/key head of V head h */",
     "const int j = h % Hqk;"),
    ("erase_sign", "const double w = b * (vt[i] - alpha * u);",
     "const double w = b * (vt[i] + alpha * u);"),
    ("transposed_state_read", "u += Si[c] * kt[c];", "u += S[(size_t)c * Dk + i] * kt[c];"),
    ("initial_state_ignored",
     "memcpy(S, J->initial_state + ((size_t)n * Hv + h) * sdim, sdim * sizeof(double));\n    else\n        memset(S, 0, sdim * sizeof(double));\n\n    for (int64_t t",
     "memset(S, 0, sdim * sizeof(double));\n    else\n        memset(S, 0, sdim * sizeof(double));\n\n    for (int64_t t"),
    ("chunk_decay_off_by_one", "a = BVAL(r) * exp(G[r] - G[s]) * kk;", "a = BVAL(r) * exp(G[r] - G[s + 1]) * kk;"),
    ("chunk_output_strict", "for (int s = 0; s <= r; ++s) {", "for (int s = 0; s < r; ++s) {"),
    ("chunk_carry_undecayed", "double x = eL * S[(size_t)i * Dk + c];", "double x = S[(size_t)i * Dk + c];"),
    ("bf16_ties_away", "const double r = nearbyint(ldexp(a, -qexp));", "const double r = round(ldexp(a, -qexp));"),
    ("bf16_truncate", "const double r = nearbyint(ldexp(a, -qexp));", "const double r = trunc(ldexp(a, -qexp));"),
    ("bf16_seven_bits", "int qexp = e - 8;", "int qexp = e - 7;"),
    ("bf16_no_subnormal_floor", "if (qexp < -133) qexp = -133;", "if (qexp < -149) qexp = -149;"),
    ("bf16_no_overflow", "if (fabs(y) > bf16_max) y = copysign(INFINITY, a);", "(void)bf16_max;"),
    ("prologue_no_sqrt", "for (int c = 0; c < Dk; ++c) x[c] /= norm;", "for (int c = 0; c < Dk; ++c) x[c] /= ss;"),
    ("prologue_l1_norm", "for (int c = 0; c < Dk; ++c) ss += x[c] * x[c];", "for (int c = 0; c < Dk; ++c) ss += fabs(x[c]);"),
    ("prologue_q_only", "for (int w = 0; w < 2; ++w) {", "for (int w = 0; w < 1; ++w) {"),
    ("prologue_relu_not_softplus", "g[i] = -(fmax(a, 0.0) + log1p(exp(-fabs(a))));", "g[i] = -(fmax(a, 0.0));"),
    ("prologue_decay_sign", "g[i] = -(fmax(a, 0.0) + log1p(exp(-fabs(a))));", "g[i] = (fmax(a, 0.0) + log1p(exp(-fabs(a))));"),
    ("bwd_carry_without_decay", "G[(size_t)i * Dk + c] = alpha * (G[(size_t)i * Dk + c] - b * Gk[i] * kt[c]);",
     "G[(size_t)i * Dk + c] = (G[(size_t)i * Dk + c] - b * Gk[i] * kt[c]);"),
    ("bwd_dk_sign", "acc += b * G[(size_t)i * Dk + c] * (vt[i] - alpha * u[i]) -",
     "acc += b * G[(size_t)i * Dk + c] * (vt[i] - alpha * u[i]) +"),
    ("bwd_dq_from_previous_state", "dqt[c] += scale * St[(size_t)i * Dk + c] * dOt[i];",
     "dqt[c] += scale * Sp[(size_t)i * Dk + c] * dOt[i];"),
    ("bwd_dg_not_chained", "dg[t * Hv + h] = alpha * (sGS - b * gku);", "dg[t * Hv + h] = (sGS - b * gku);"),
    ("bwd_dbeta_without_decay", "wgk += (vt[i] - alpha * ui) * gk;", "wgk += (vt[i] - ui) * gk;"),
    ("prologue_sigmoid_of_minus_b", "beta[i] = b >= 0.0 ? 1.0 / (1.0 + exp(-b)) : exp(b) / (1.0 + exp(b));",
     "beta[i] = b >= 0.0 ? 1.0 / (1.0 + exp(b)) : exp(-b) / (1.0 + exp(-b));"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new, 1)
    path = tmp_path / "mut.c"
    path.write_text(mutated)
    so = str(tmp_path / f"libmut_{name}.so")
    oracle.build(src=str(path), out=so)
    lib = oracle.load(so)
    caught = []
    for check in P.ALL_CHECKS:
        try:
            check(lib)
        except (AssertionError, ValueError, FloatingPointError) as e:
            caught.append((check.__name__, str(e)[:80]))
    assert caught, f"no pin catches mutant {name}"
