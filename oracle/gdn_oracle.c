/*
 * gdn_oracle.c -- plain fp64 CPU oracle for the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The CUDA library
 * never calls it and shares no code, header or constant with it.
 *
 * What it computes (the definition, written out token by token):
 *
 *   S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *   o_t = scale * S_t q_t
 *
 * Source: "Inside Qwen3.8-27B: Hybrid DeltaNet Architecture, 256k Context,
 * and 24GB Local Serving", section "Gated DeltaNet Mechanics" (the delta rule
 * removes the old association stored under k_t before writing v_t; S_t is a
 * d x d state of fixed size; k_t is the normalized key, v_t the value).  The
 * displayed equation did not survive on that page; the form above is the
 * gated delta rule it describes in words, with alpha_t = exp(g_t) the decay
 * and beta_t the write strength.  Head layout (16 query/key heads shared by
 * 48 value heads, head dim 128): "Qwen 3.8 27B Review: Native Vision, FP8
 * Quantization & 1M Context in a Compact Dense Model", section "3.
 * Architecture: Gated DeltaNet Hybrid + FP8 Quantization".
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes of the repository):
 *   - S is stored Dv x Dk (row i = value dimension i, Dk contiguous), so the
 *     write term is v k^T, the read is S k and the output is S q.
 *   - V head h reads query/key head h / (Hv / Hqk) (contiguous groups).
 *   - g and beta are per (token, V head); alpha = exp(g).
 *   - o_t uses the state after token t's update.
 *   - Each sequence starts from its own initial state (zeros if none).
 *
 * The update is applied row by row: with u = S_{t-1} k_t (one number per
 * row i of S),  alpha S (I - beta k k^T) + beta v k^T
 *             = alpha S + beta (v - alpha u) k^T,
 * which touches row i of S only through u_i.  That identity is the only
 * rearrangement here; it is exact algebra, and the tests check the result
 * against the explicit matrix-product form computed independently.
 *
 * Also here: the chunked (WY / UT-transform) form of the same recurrence,
 * derived from the definition above, in fp64.  It exists to show that the
 * chunked algebra a GPU kernel follows reproduces the token-by-token
 * definition; the tests check it against the sequential oracle.
 *
 * Threads: units (sequence, V head) are independent and are spread over
 * POSIX threads; inside a unit the arithmetic order is fixed, so results do
 * not depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NO_MEMORY 2

typedef struct {
    const double *q, *k, *v, *g, *beta;
    const int64_t *cu_seqlens;
    int num_seqs, Hqk, Hv, Dk, Dv, chunk;
    double scale;
    const double *initial_state; /* [N, Hv, Dv, Dk] or NULL */
    double *final_state;         /* [N, Hv, Dv, Dk] or NULL */
    double *o;                   /* [T, Hv, Dv] */
    int64_t next_unit;           /* shared work counter */
    pthread_mutex_t lock;
    int failed;
} job_t;

/* ---- sequential definition, one (sequence n, V head h) unit ---------- */
static void sequential_unit(const job_t *J, int n, int h, double *S)
{
    const int Dk = J->Dk, Dv = J->Dv, Hqk = J->Hqk, Hv = J->Hv;
    const int j = h / (Hv / Hqk); /* query/key head of V head h */
    const size_t sdim = (size_t)Dv * Dk;

    if (J->initial_state)
        memcpy(S, J->initial_state + ((size_t)n * Hv + h) * sdim, sdim * sizeof(double));
    else
        memset(S, 0, sdim * sizeof(double));

    for (int64_t t = J->cu_seqlens[n]; t < J->cu_seqlens[n + 1]; ++t) {
        const double alpha = exp(J->g[t * Hv + h]);
        const double b = J->beta[t * Hv + h];
        const double *kt = J->k + ((size_t)t * Hqk + j) * Dk;
        const double *qt = J->q + ((size_t)t * Hqk + j) * Dk;
        const double *vt = J->v + ((size_t)t * Hv + h) * Dv;
        double *ot = J->o + ((size_t)t * Hv + h) * Dv;

        for (int i = 0; i < Dv; ++i) {
            double *Si = S + (size_t)i * Dk;
            double u = 0.0; /* u_i = (S_{t-1} k_t)_i */
            for (int c = 0; c < Dk; ++c) u += Si[c] * kt[c];
            const double w = b * (vt[i] - alpha * u);
            for (int c = 0; c < Dk; ++c) Si[c] = alpha * Si[c] + w * kt[c];
        }
        for (int i = 0; i < Dv; ++i) {
            const double *Si = S + (size_t)i * Dk;
            double acc = 0.0; /* (S_t q_t)_i */
            for (int c = 0; c < Dk; ++c) acc += Si[c] * qt[c];
            ot[i] = J->scale * acc;
        }
    }
    if (J->final_state)
        memcpy(J->final_state + ((size_t)n * Hv + h) * sdim, S, sdim * sizeof(double));
}

/* ---- chunked WY / UT form, one unit ----------------------------------
 *
 * Within a chunk of C' <= C tokens (aligned to the sequence start) with
 * start state S0 and local prefix sums G_t = g_1 + ... + g_t:
 *   writing w_t = beta_t (v_t - alpha_t S_{t-1} k_t), S_t = alpha_t S_{t-1} + w_t k_t^T,
 *   S_t = e^{G_t} S0 + sum_{s<=t} e^{G_t-G_s} w_s k_s^T.
 * Substituting into w_t gives the unit lower-triangular system
 *   w_t + sum_{s<t} A_ts w_s = beta_t (v_t - e^{G_t} S0 k_t),
 *   A_ts = beta_t e^{G_t-G_s} (k_t . k_s),
 * so with Tm = (I + A)^{-1}:  W = Tm diag(beta e^G) K,  Ut = Tm diag(beta) V,
 *   U = Ut - W S0^T            (row t of U is w_t),
 *   o_t = e^{G_t} S0 q_t + sum_{s<=t} e^{G_t-G_s} (q_t . k_s) w_s,
 *   S_C' = e^{G_C'} S0 + sum_s e^{G_C'-G_s} w_s k_s^T.
 * Requires finite g (exp(G_t - G_s) of two infinite sums is undefined).
 */
static void chunked_unit(const job_t *J, int n, int h, double *S, double *scratch)
{
    const int Dk = J->Dk, Dv = J->Dv, Hqk = J->Hqk, Hv = J->Hv, C = J->chunk;
    const int j = h / (Hv / Hqk);
    const size_t sdim = (size_t)Dv * Dk;
    double *G = scratch;                       /* C       */
    double *A = G + C;                         /* C x C   */
    double *Tm = A + (size_t)C * C;            /* C x C   */
    double *W = Tm + (size_t)C * C;            /* C x Dk  */
    double *U = W + (size_t)C * Dk;            /* C x Dv  */
    double *Snew = U + (size_t)C * Dv;         /* Dv x Dk */

    if (J->initial_state)
        memcpy(S, J->initial_state + ((size_t)n * Hv + h) * sdim, sdim * sizeof(double));
    else
        memset(S, 0, sdim * sizeof(double));

    const int64_t t0 = J->cu_seqlens[n], t1 = J->cu_seqlens[n + 1];
    for (int64_t c0 = t0; c0 < t1; c0 += C) {
        const int L = (int)((t1 - c0) < C ? (t1 - c0) : C);
#define KROW(r) (J->k + ((size_t)(c0 + (r)) * Hqk + j) * Dk)
#define QROW(r) (J->q + ((size_t)(c0 + (r)) * Hqk + j) * Dk)
#define VROW(r) (J->v + ((size_t)(c0 + (r)) * Hv + h) * Dv)
#define GVAL(r) (J->g[(c0 + (r)) * Hv + h])
#define BVAL(r) (J->beta[(c0 + (r)) * Hv + h])
        double acc = 0.0;
        for (int r = 0; r < L; ++r) { acc += GVAL(r); G[r] = acc; }

        /* A (strictly lower) */
        for (int r = 0; r < L; ++r)
            for (int s = 0; s < L; ++s) {
                double a = 0.0;
                if (s < r) {
                    double kk = 0.0;
                    for (int c = 0; c < Dk; ++c) kk += KROW(r)[c] * KROW(s)[c];
                    a = BVAL(r) * exp(G[r] - G[s]) * kk;
                }
                A[(size_t)r * C + s] = a;
            }
        /* Tm = (I + A)^{-1} by forward substitution, column by column */
        for (int col = 0; col < L; ++col)
            for (int r = 0; r < L; ++r) {
                double x = (r == col) ? 1.0 : 0.0;
                for (int s = 0; s < r; ++s) x -= A[(size_t)r * C + s] * Tm[(size_t)s * C + col];
                Tm[(size_t)r * C + col] = x;
            }
        /* W = Tm diag(beta e^G) K ;  U = Tm diag(beta) V - W S0^T */
        for (int r = 0; r < L; ++r) {
            for (int c = 0; c < Dk; ++c) {
                double x = 0.0;
                for (int s = 0; s < L; ++s) x += Tm[(size_t)r * C + s] * BVAL(s) * exp(G[s]) * KROW(s)[c];
                W[(size_t)r * Dk + c] = x;
            }
            for (int i = 0; i < Dv; ++i) {
                double x = 0.0;
                for (int s = 0; s < L; ++s) x += Tm[(size_t)r * C + s] * BVAL(s) * VROW(s)[i];
                double ws = 0.0;
                for (int c = 0; c < Dk; ++c) ws += W[(size_t)r * Dk + c] * S[(size_t)i * Dk + c];
                U[(size_t)r * Dv + i] = x - ws;
            }
        }
        /* outputs */
        for (int r = 0; r < L; ++r) {
            double *ot = J->o + ((size_t)(c0 + r) * Hv + h) * Dv;
            const double er = exp(G[r]);
            for (int i = 0; i < Dv; ++i) {
                double x = 0.0;
                for (int c = 0; c < Dk; ++c) x += S[(size_t)i * Dk + c] * QROW(r)[c];
                x *= er;
                for (int s = 0; s <= r; ++s) {
                    double qk = 0.0;
                    for (int c = 0; c < Dk; ++c) qk += QROW(r)[c] * KROW(s)[c];
                    x += exp(G[r] - G[s]) * qk * U[(size_t)s * Dv + i];
                }
                ot[i] = J->scale * x;
            }
        }
        /* carried state */
        const double eL = exp(G[L - 1]);
        for (int i = 0; i < Dv; ++i)
            for (int c = 0; c < Dk; ++c) {
                double x = eL * S[(size_t)i * Dk + c];
                for (int s = 0; s < L; ++s) x += exp(G[L - 1] - G[s]) * U[(size_t)s * Dv + i] * KROW(s)[c];
                Snew[(size_t)i * Dk + c] = x;
            }
        memcpy(S, Snew, sdim * sizeof(double));
#undef KROW
#undef QROW
#undef VROW
#undef GVAL
#undef BVAL
    }
    if (J->final_state)
        memcpy(J->final_state + ((size_t)n * Hv + h) * sdim, S, sdim * sizeof(double));
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const size_t sdim = (size_t)J->Dv * J->Dk;
    size_t extra = 0;
    if (J->chunk > 0)
        extra = (size_t)J->chunk * (1 + 2 * (size_t)J->chunk + J->Dk + J->Dv) + sdim;
    double *S = (double *)malloc((sdim + extra) * sizeof(double));
    if (!S) {
        pthread_mutex_lock(&J->lock);
        J->failed = 1;
        pthread_mutex_unlock(&J->lock);
        return NULL;
    }
    const int64_t total = (int64_t)J->num_seqs * J->Hv;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int64_t u = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (u >= total) break;
        const int n = (int)(u / J->Hv), h = (int)(u % J->Hv);
        if (J->chunk > 0)
            chunked_unit(J, n, h, S, S + sdim);
        else
            sequential_unit(J, n, h, S);
    }
    free(S);
    return NULL;
}

static int run(job_t *J, int num_threads)
{
    if (!J->q || !J->k || !J->v || !J->g || !J->beta || !J->cu_seqlens || !J->o) return ORACLE_BAD_ARG;
    if (J->num_seqs < 0 || J->Hqk <= 0 || J->Hv <= 0 || J->Dk <= 0 || J->Dv <= 0) return ORACLE_BAD_ARG;
    if (J->Hv % J->Hqk != 0) return ORACLE_BAD_ARG;
    if (J->cu_seqlens[0] != 0) return ORACLE_BAD_ARG;
    for (int n = 0; n < J->num_seqs; ++n)
        if (J->cu_seqlens[n + 1] < J->cu_seqlens[n]) return ORACLE_BAD_ARG;

    if (num_threads <= 0) num_threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (num_threads <= 0) num_threads = 1;
    const int64_t units = (int64_t)J->num_seqs * J->Hv;
    if (num_threads > units) num_threads = (int)(units > 0 ? units : 1);

    J->next_unit = 0;
    J->failed = 0;
    pthread_mutex_init(&J->lock, NULL);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)num_threads);
    if (!th) { pthread_mutex_destroy(&J->lock); return ORACLE_NO_MEMORY; }
    int started = 0;
    for (int i = 0; i < num_threads; ++i) {
        if (pthread_create(&th[i], NULL, worker, J) != 0) break;
        ++started;
    }
    if (started == 0) worker(J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J->lock);
    return J->failed ? ORACLE_NO_MEMORY : ORACLE_OK;
}

/*
 * Prefill over packed sequences.  Arrays are host fp64, row-major:
 *   q, k [T, Hqk, Dk];  v [T, Hv, Dv];  g, beta [T, Hv];  o [T, Hv, Dv];
 *   cu_seqlens [num_seqs + 1] (cu_seqlens[0] = 0, non-decreasing, last = T);
 *   initial_state, final_state [num_seqs, Hv, Dv, Dk] (either may be NULL;
 *   NULL initial state means zeros, NULL final state skips the write).
 * chunk = 0 runs the token-by-token definition; chunk > 0 runs the chunked
 * WY/UT form with that chunk size.  num_threads <= 0 uses every online core.
 * Returns 0 on success, 1 on a bad argument, 2 when memory ran out.
 */
int gdn_oracle_prefill(const double *q, const double *k, const double *v, const double *g,
                       const double *beta, const int64_t *cu_seqlens, int num_seqs, int Hqk,
                       int Hv, int Dk, int Dv, double scale, const double *initial_state,
                       double *final_state, double *o, int chunk, int num_threads)
{
    job_t J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.cu_seqlens = cu_seqlens;
    J.num_seqs = num_seqs; J.Hqk = Hqk; J.Hv = Hv; J.Dk = Dk; J.Dv = Dv; J.chunk = chunk;
    J.scale = scale; J.initial_state = initial_state; J.final_state = final_state; J.o = o;
    if (chunk < 0) return ORACLE_BAD_ARG;
    return run(&J, num_threads);
}

/*
 * One decode step for B sequences, one token each: the same update as the
 * prefill applied once per (sequence b, V head h), state updated in place.
 *   q, k [B, Hqk, Dk];  v [B, Hv, Dv];  g, beta [B, Hv];  state [B, Hv, Dv, Dk];
 *   o [B, Hv, Dv].
 */
int gdn_oracle_decode_step(const double *q, const double *k, const double *v, const double *g,
                           const double *beta, double *state, double *o, int B, int Hqk, int Hv,
                           int Dk, int Dv, double scale, int num_threads)
{
    if (B < 0) return ORACLE_BAD_ARG;
    int64_t *cu = (int64_t *)malloc(sizeof(int64_t) * ((size_t)B + 1));
    if (!cu) return ORACLE_NO_MEMORY;
    for (int b = 0; b <= B; ++b) cu[b] = b; /* B sequences of one token each */
    int rc = gdn_oracle_prefill(q, k, v, g, beta, cu, B, Hqk, Hv, Dk, Dv, scale, state, state, o,
                                0, num_threads);
    free(cu);
    return rc;
}

/*
 * States kept at rest in bf16: round each x[i] to the nearest value of the
 * bf16 format, ties to even, straight from fp64 (one rounding, no fp32 step).
 * bf16 keeps 8 significant bits and the exponent range of IEEE binary32: in
 * the binade [2^(e-1), 2^e) its values are the multiples of 2^(e-8); below
 * 2^-126 (subnormals) the multiples of 2^-133; the largest finite value is
 * (2 - 2^-7) 2^127, and a value that rounds above it becomes infinite.  This
 * is IEEE 754 round-to-nearest-even applied to that format, written out.
 * Returns 0, or 1 for a bad argument.
 */
int gdn_oracle_round_bf16(double *x, int64_t n)
{
    if (n < 0 || (n > 0 && !x)) return ORACLE_BAD_ARG;
    const double bf16_max = ldexp(255.0, 120); /* (2 - 2^-7) 2^127 */
    for (int64_t i = 0; i < n; ++i) {
        const double a = x[i];
        if (!isfinite(a) || a == 0.0) continue;
        int e;
        frexp(a, &e); /* a = m 2^e with 0.5 <= |m| < 1 */
        int qexp = e - 8;
        if (qexp < -133) qexp = -133;
        const double r = nearbyint(ldexp(a, -qexp)); /* default rounding mode: ties to even */
        double y = ldexp(r, qexp);
        if (fabs(y) > bf16_max) y = copysign(INFINITY, a);
        x[i] = y;
    }
    return ORACLE_OK;
}

/*
 * Input prologue: from the layer's raw projections to the inputs of the
 * recurrence, in place.  "Inside Qwen3.8-27B ...", section "Gated DeltaNet
 * Mechanics", calls k_t the normalized key projection and makes beta_t input
 * dependent; the maps below are the plainest readings (listed in the design
 * notes of the repository):
 *   q_t, k_t  <- x / |x|_2 for each (token, query/key head) row of Dk values;
 *                a row of zeros stays zero;
 *   g_t       <- -softplus(a_t) = -log(1 + e^{a_t}), so alpha_t = e^{g_t} lies in (0, 1);
 *   beta_t    <- sigmoid(b_t) = 1 / (1 + e^{-b_t}), in (0, 1).
 * On entry g and beta hold a and b ([T, Hv]); q and k are [T, Hqk, Dk].
 * Returns 0, or 1 for a bad argument.
 */
int gdn_oracle_prologue(double *q, double *k, double *g, double *beta, int64_t T, int Hqk, int Hv,
                        int Dk)
{
    if (T < 0 || Hqk <= 0 || Hv <= 0 || Dk <= 0) return ORACLE_BAD_ARG;
    if (T > 0 && (!q || !k || !g || !beta)) return ORACLE_BAD_ARG;
    double *rows[2] = {q, k};
    for (int w = 0; w < 2; ++w) {
        for (int64_t r = 0; r < T * Hqk; ++r) {
            double *x = rows[w] + r * Dk;
            double ss = 0.0;
            for (int c = 0; c < Dk; ++c) ss += x[c] * x[c];
            if (ss == 0.0) continue;
            const double norm = sqrt(ss);
            for (int c = 0; c < Dk; ++c) x[c] /= norm;
        }
    }
    for (int64_t i = 0; i < T * Hv; ++i) {
        const double a = g[i], b = beta[i];
        /* softplus(a) = max(a, 0) + log(1 + e^{-|a|}), the same value without overflow */
        g[i] = -(fmax(a, 0.0) + log1p(exp(-fabs(a))));
        beta[i] = b >= 0.0 ? 1.0 / (1.0 + exp(-b)) : exp(b) / (1.0 + exp(b));
    }
    return ORACLE_OK;
}

/*
 * Backward pass (reverse-mode derivative) of the recurrence, token by token.
 * The forward definition is the one above; the loss L is linear in the
 * outputs it is given gradients for: dO = dL/do [T, Hv, Dv] and, optionally,
 * dSfin = dL/dS_final [N, Hv, Dv, Dk].  Writing G for dL/dS_t (everything that
 * depends on S_t), u = S_{t-1} k_t, w = v_t - alpha_t u, so that
 * S_t = alpha_t S_{t-1} + beta_t w k_t^T and o_t = scale S_t q_t, the chain
 * rule gives, for t from the last token down to the first:
 *   G      += scale dO_t q_t^T
 *   dq_t    = scale S_t^T dO_t
 *   dv_t    = beta_t G k_t
 *   dbeta_t = w . (G k_t)
 *   dg_t    = alpha_t ( <G, S_{t-1}> - beta_t (G k_t) . u )       (alpha = e^g)
 *   dk_t    = beta_t G^T w - alpha_t beta_t S_{t-1}^T (G k_t)
 *   G      <- alpha_t (G - beta_t (G k_t) k_t^T)                  (= dL/dS_{t-1})
 * and dS0 = G at the start of the sequence.  dq and dk of a query/key head
 * sum over the value heads that read it.  All states S_0 .. S_L of a unit are
 * kept (fp64), so this is for small inputs.  Outputs dq, dk [T, Hqk, Dk],
 * dv [T, Hv, Dv], dg, dbeta [T, Hv], dS0 [N, Hv, Dv, Dk] (may be NULL).
 * Returns 0, 1 for a bad argument, 2 when memory ran out.
 */
int gdn_oracle_backward(const double *q, const double *k, const double *v, const double *g,
                        const double *beta, const int64_t *cu_seqlens, int num_seqs, int Hqk,
                        int Hv, int Dk, int Dv, double scale, const double *initial_state,
                        const double *dO, const double *dSfin, double *dq, double *dk,
                        double *dv, double *dg, double *dbeta, double *dS0)
{
    if (num_seqs < 0 || Hqk <= 0 || Hv <= 0 || Hv % Hqk || Dk <= 0 || Dv <= 0) return ORACLE_BAD_ARG;
    const int64_t T = cu_seqlens[num_seqs];
    const size_t sdim = (size_t)Dv * Dk;
    memset(dq, 0, sizeof(double) * (size_t)T * Hqk * Dk);
    memset(dk, 0, sizeof(double) * (size_t)T * Hqk * Dk);
    int64_t Lmax = 0;
    for (int n = 0; n < num_seqs; ++n) {
        const int64_t L = cu_seqlens[n + 1] - cu_seqlens[n];
        if (L < 0) return ORACLE_BAD_ARG;
        if (L > Lmax) Lmax = L;
    }
    double *states = (double *)malloc(sizeof(double) * sdim * (size_t)(Lmax + 1));
    double *G = (double *)malloc(sizeof(double) * sdim);
    double *Gk = (double *)malloc(sizeof(double) * Dv);
    double *u = (double *)malloc(sizeof(double) * Dv);
    if (!states || !G || !Gk || !u) {
        free(states); free(G); free(Gk); free(u);
        return ORACLE_NO_MEMORY;
    }
    for (int n = 0; n < num_seqs; ++n) {
        const int64_t t0 = cu_seqlens[n], L = cu_seqlens[n + 1] - t0;
        for (int h = 0; h < Hv; ++h) {
            const int j = h / (Hv / Hqk);
            /* forward, keeping S_0 .. S_L */
            if (initial_state) memcpy(states, initial_state + ((size_t)n * Hv + h) * sdim, sdim * sizeof(double));
            else memset(states, 0, sdim * sizeof(double));
            for (int64_t s = 0; s < L; ++s) {
                const int64_t t = t0 + s;
                const double alpha = exp(g[t * Hv + h]), b = beta[t * Hv + h];
                const double *kt = k + ((size_t)t * Hqk + j) * Dk, *vt = v + ((size_t)t * Hv + h) * Dv;
                const double *Sp = states + (size_t)s * sdim;
                double *Sn = states + (size_t)(s + 1) * sdim;
                for (int i = 0; i < Dv; ++i) {
                    double ui = 0.0;
                    for (int c = 0; c < Dk; ++c) ui += Sp[(size_t)i * Dk + c] * kt[c];
                    const double wi = b * (vt[i] - alpha * ui);
                    for (int c = 0; c < Dk; ++c) Sn[(size_t)i * Dk + c] = alpha * Sp[(size_t)i * Dk + c] + wi * kt[c];
                }
            }
            /* backward */
            if (dSfin) memcpy(G, dSfin + ((size_t)n * Hv + h) * sdim, sdim * sizeof(double));
            else memset(G, 0, sdim * sizeof(double));
            for (int64_t s = L - 1; s >= 0; --s) {
                const int64_t t = t0 + s;
                const double alpha = exp(g[t * Hv + h]), b = beta[t * Hv + h];
                const double *kt = k + ((size_t)t * Hqk + j) * Dk, *qt = q + ((size_t)t * Hqk + j) * Dk;
                const double *vt = v + ((size_t)t * Hv + h) * Dv, *dOt = dO + ((size_t)t * Hv + h) * Dv;
                const double *Sp = states + (size_t)s * sdim, *St = states + (size_t)(s + 1) * sdim;
                double *dqt = dq + ((size_t)t * Hqk + j) * Dk, *dkt = dk + ((size_t)t * Hqk + j) * Dk;
                /* o_t = scale S_t q_t */
                for (int i = 0; i < Dv; ++i)
                    for (int c = 0; c < Dk; ++c) {
                        G[(size_t)i * Dk + c] += scale * dOt[i] * qt[c];
                        dqt[c] += scale * St[(size_t)i * Dk + c] * dOt[i];
                    }
                double sGS = 0.0, gku = 0.0, wgk = 0.0;
                for (int i = 0; i < Dv; ++i) {
                    double gk = 0.0, ui = 0.0;
                    for (int c = 0; c < Dk; ++c) {
                        gk += G[(size_t)i * Dk + c] * kt[c];
                        ui += Sp[(size_t)i * Dk + c] * kt[c];
                        sGS += G[(size_t)i * Dk + c] * Sp[(size_t)i * Dk + c];
                    }
                    Gk[i] = gk;
                    u[i] = ui;
                    gku += gk * ui;
                    wgk += (vt[i] - alpha * ui) * gk;
                }
                for (int i = 0; i < Dv; ++i) dv[((size_t)t * Hv + h) * Dv + i] = b * Gk[i];
                dbeta[t * Hv + h] = wgk;
                dg[t * Hv + h] = alpha * (sGS - b * gku);
                for (int c = 0; c < Dk; ++c) {
                    double acc = 0.0;
                    for (int i = 0; i < Dv; ++i)
                        acc += b * G[(size_t)i * Dk + c] * (vt[i] - alpha * u[i]) -
                               alpha * b * Sp[(size_t)i * Dk + c] * Gk[i];
                    dkt[c] += acc;
                }
                for (int i = 0; i < Dv; ++i)
                    for (int c = 0; c < Dk; ++c)
                        G[(size_t)i * Dk + c] = alpha * (G[(size_t)i * Dk + c] - b * Gk[i] * kt[c]);
            }
            if (dS0) memcpy(dS0 + ((size_t)n * Hv + h) * sdim, G, sdim * sizeof(double));
        }
    }
    free(states); free(G); free(Gk); free(u);
    return ORACLE_OK;
}
