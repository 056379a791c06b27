// gdn_backward_chunked.cu -- backward pass of the gated delta rule in the
// chunked (WY/UT) form: the gradients of a loss with respect to q, k, v, g,
// beta and the initial state, fp32-accurate, with the dense products of every
// chunk on the tensor cores.
//
// The forward rule is the one of "Inside Qwen3.8-27B: Hybrid DeltaNet
// Architecture, 256k Context, and 24GB Local Serving", section "Gated DeltaNet
// Mechanics", whose note says the block-parallel form serves training as well
// as prefill.  For a chunk of C = 64 tokens with start state S0 (Dv x Dk),
// local log-decay prefix sums G_t, gamma_t = e^{G_t}, kdec_t = e^{G_last -
// G_t}, gamma_C = e^{G_last} and E_ts = e^{G_t - G_s} (s <= t):
//   A = strict_lower(diag(beta) (E . K K^T)),   Tm = (I + A)^-1
//   W = Tm diag(beta gamma) K,   U~ = Tm diag(beta) V,   U = U~ - W S0^T
//   P = E . Q K^T (s <= t),      O = scale (diag(gamma) Q S0^T + P U)
//   S1 = gamma_C S0 + U^T diag(kdec) K
// Reverse mode, with dO' = scale dO and dS1 = dL/dS1 (the state after the
// chunk), first the chain over the chunks, last to first:
//   dU  = P^T dO' + diag(kdec) K dS1^T
//   dS0 = gamma_C dS1 + dO'^T diag(gamma) Q - dU^T W
// then, for every chunk independently:
//   dQ  = diag(gamma) dO' S0 + (dP . E) K,        dP = lower(dO' U^T)
//   dW  = -dU S0,   dT = dW (diag(beta gamma) K)^T + dU (diag(beta) V)^T
//   X = Tm^T dW,    Y = Tm^T dU,                  dA = strict_lower(-Tm^T dT Tm^T)
//   dK  = diag(kdec) U dS1 + (dP . E)^T Q + diag(beta gamma) X + (B + B^T) K,
//         B = diag(beta) (dA . E)
//   dV  = diag(beta) Y
//   dbeta_t = gamma_t X_t.k_t + Y_t.v_t + sum_s dA_ts (E . K K^T)_ts
//   dG_t from every e^{G} factor (gamma, kdec, gamma_C, E in P and A), and
//   dg_s = sum_{t >= s} dG_t within the chunk.
// dq and dk of a query/key head sum over the value heads that read it.
//
// Launches (one stream):
//   plan         validates cu_seqlens, lists the non-empty sequences and
//                their first chunk; d_initial_state of an empty sequence is
//                d_final_state (or zero)
//   prep         per (chunk, value head): P, E . K K^T, Tm, W, U~, G
//   chains       one launch of both chains, which do not depend on each
//                other: per (sequence, value head, 64 state rows) the reverse
//                one (dS1 and dU per chunk, last to first, and
//                d_initial_state), then per (sequence, value head) the
//                forward one (the state at every chunk start S0, and U)
//   grads_state  per (chunk, value head): the products with S0 and dS1
//   grads_local  per (chunk, query/key head), its value heads in turn: the
//                64 x 64 algebra, dv, dg, dbeta, and dq, dk summed over the
//                group in registers (fixed order)
// Rows of S and of dS evolve independently (the chains never mix rows), so a
// reverse-chain CTA owns 64 of the Dv rows.  Tiles move global -> shared with
// cp.async, all of a step's copies in flight at once, and the chains fetch a
// chunk's tiles while the previous chunk computes where buffers allow.
// Products run on tensor cores at about fp32 accuracy: fp32 operands split
// into hi and lo parts and three products hi*hi + hi*lo + lo*hi, a raw bf16
// input used as it is (its lo part is zero).  The state gradients run on
// tcgen05 (bf16 hi/lo images, TMEM accumulators); the rest on warp-level MMAs,
// m16n8k16 bf16 where an operand is a raw bf16 input, m16n8k8 tf32 otherwise.  Per-row sums go through fixed-order partials, so results do
// not depend on scheduling.
#include <algorithm>

#include "gdn_chunk_ops.cuh"
#include "gdn_common.cuh"
#include "gdn_twophase.cuh"

namespace gdn {

cudaError_t launch_plan(const int32_t *cu, int N, int T, int Hv, const void *s0, void *sfin,
                        size_t state_bytes, tp::PlanHeader *ph, int32_t *ne_seq, int32_t *ne_cs,
                        int32_t *status, cudaStream_t stream);

namespace cbwd {

constexpr int C = 64;         // chunk length
constexpr int NT = 256;       // threads per CTA (8 warps)
constexpr int NTR = 512;      // threads of a reverse-chain CTA (16 warps: one CTA per SM)
constexpr int SL = 64;        // state rows per chain CTA
constexpr int LD64 = 68;      // fp32 row stride of 64 x 64 tiles in shared memory
constexpr float kGmin = -30.f;  // g clamp: alpha >= e^-30, so prefix sums stay finite

struct Params {
  const void *q, *k, *v;
  const float *g, *beta;
  const int32_t *cu;
  int N, T, Hqk, Hv;
  float scale;
  const float *s0, *dO, *dSf;
  float *dq, *dk;  // [T, Hqk, Dk] outputs
  float *dv, *dg, *dbeta, *ds0;
  const tp::PlanHeader *ph;
  const int32_t *ne_seq, *ne_cs;
  // per unit u = chunk * Hv + value head
  float *Tm, *P, *EKK;      // [u][64][64]
  float *W, *dQp, *dKp, *dW;  // [u][64][Dk]
  float *Ut, *U, *dU;       // [u][64][Dv]
  float *S0, *dS1;          // [u][Dv][Dk]
  double *G;                // [u][64] prefix sums of the clamped log-decays (fp64: differences
                            // of large sums stay exact when gates are near zero)
  float *sc;                // [u][3][64]: dgamma (from S0), dkdec, dgamma_C at [2][0]
  int32_t *status;          // workspace header: status word, then the wait limit
};

// ---- tensor-core building block -------------------------------------------
// Warp-level m16n8k16 bf16 MMA with fp32 accumulation.
__device__ __forceinline__ void mma_bf16_16x8x16(float *d, const uint32_t *a, const uint32_t *b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// Split of two fp32 values into packed bf16 pairs hi = bf16(x) and lo =
// bf16(x - hi), both rounded to nearest: |x - hi - lo| <= 2^-18 |x|.
__device__ __forceinline__ void split2(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}

// Split of an fp32 value for the 3-term tf32 products: hi keeps the sign,
// exponent and the 10 mantissa bits a tf32 operand holds (the low 13 bits
// cleared, |x - hi| < 2^-10 |x|); lo = x - hi is exact in fp32 and goes to the
// MMA as is, which reads only its tf32 bits (|error| < 2^-10 |lo|).  So
// hi*hi' + hi*lo' + lo*hi' is within about 2^-18 of x*y.
__device__ __forceinline__ uint32_t tf32_hi(float x) { return __float_as_uint(x) & 0xffffe000u; }
__device__ __forceinline__ uint32_t tf32_lo(float x, uint32_t hi) {
  return __float_as_uint(x - __uint_as_float(hi));
}

// acc[t] (a 16 x 8 fragment) += X[16][KDIM] * Y[KDIM][8 t .. 8 t + 7] for t <
// NTL tiles in a row, on warp-level tensor-core MMAs.  X(r, c) and Y(r, c)
// read single elements; each is split once per k step.  Fragment element e
// of tile t sits at row gid + 8 (e >> 1), column 8 t + 2 tig + (e & 1) (gid =
// lane / 4, tig = lane % 4) for both MMA shapes used:
//   - an operand marked exact holds bf16 values already (a raw bf16 input):
//     m16n8k16 bf16 MMAs, the other operand split into bf16 hi + lo (rounded
//     to nearest, |x - hi - lo| <= 2^-18 |x|): two MMAs per k step, one when
//     both operands are exact;
//   - otherwise m16n8k8 tf32 MMAs with both operands split (tf32_hi, tf32_lo)
//     and three products per k step.
template <int KDIM, int NTL, bool XEXACT = false, bool YEXACT = false, class FX, class FY>
__device__ __forceinline__ void mma3_rows(float (&acc)[NTL][4], FX X, FY Y, int lane) {
  const int gid = lane >> 2, tig = lane & 3;
  if constexpr (XEXACT || YEXACT) {
#pragma unroll 2
    for (int ks = 0; ks < KDIM / 16; ++ks) {
      const int k0 = 16 * ks + 2 * tig;
      uint32_t ah[4], al[4];
      split2(X(gid, k0), X(gid, k0 + 1), ah[0], al[0]);
      split2(X(gid + 8, k0), X(gid + 8, k0 + 1), ah[1], al[1]);
      split2(X(gid, k0 + 8), X(gid, k0 + 9), ah[2], al[2]);
      split2(X(gid + 8, k0 + 8), X(gid + 8, k0 + 9), ah[3], al[3]);
#pragma unroll
      for (int t = 0; t < NTL; ++t) {
        const int n = 8 * t + gid;
        uint32_t bh[2], bl[2];
        split2(Y(k0, n), Y(k0 + 1, n), bh[0], bl[0]);
        split2(Y(k0 + 8, n), Y(k0 + 9, n), bh[1], bl[1]);
        if (!XEXACT) mma_bf16_16x8x16(acc[t], al, bh);
        if (!YEXACT) mma_bf16_16x8x16(acc[t], ah, bl);
        mma_bf16_16x8x16(acc[t], ah, bh);
      }
    }
  } else {
#pragma unroll 2
    for (int ks = 0; ks < KDIM / 8; ++ks) {
      const int k0 = 8 * ks + tig;
      const float a[4] = {X(gid, k0), X(gid + 8, k0), X(gid, k0 + 4), X(gid + 8, k0 + 4)};
      uint32_t ah[4], al[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ah[e] = tf32_hi(a[e]);
        al[e] = tf32_lo(a[e], ah[e]);
      }
#pragma unroll
      for (int t = 0; t < NTL; ++t) {
        const float b0 = Y(k0, 8 * t + gid), b1 = Y(k0 + 4, 8 * t + gid);
        const uint32_t bh[2] = {tf32_hi(b0), tf32_hi(b1)};
        const uint32_t bl[2] = {tf32_lo(b0, bh[0]), tf32_lo(b1, bh[1])};
        chunk::mma_tf32_16x8x8(acc[t], al, bh);
        chunk::mma_tf32_16x8x8(acc[t], ah, bl);
        chunk::mma_tf32_16x8x8(acc[t], ah, bh);
      }
    }
  }
}

template <int NTL>
__device__ __forceinline__ void zero_acc(float (&acc)[NTL][4]) {
#pragma unroll
  for (int t = 0; t < NTL; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
}

// Call f(row, col, value&) for every element of a lane's fragments; rows from
// r0, columns from c0.
template <int NTL, class F>
__device__ __forceinline__ void for_frag(float (&acc)[NTL][4], int r0, int c0, int lane, F f) {
  const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int t = 0; t < NTL; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) f(r0 + gid + 8 * (e >> 1), c0 + 8 * t + 2 * tig + (e & 1), acc[t][e]);
}

// Fragment-position loads and stores of an fp32 matrix M (row stride ld):
// the two adjacent columns a lane holds per row go as one 8-byte access.
template <int NTL>
__device__ __forceinline__ void frag_ld(float (&dst)[NTL][4], const float *M, size_t ld, int r0, int c0,
                                        int lane) {
  const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int t = 0; t < NTL; ++t) {
    const float2 a = *reinterpret_cast<const float2 *>(M + (size_t)(r0 + gid) * ld + c0 + 8 * t + 2 * tig);
    const float2 b = *reinterpret_cast<const float2 *>(M + (size_t)(r0 + gid + 8) * ld + c0 + 8 * t + 2 * tig);
    dst[t][0] = a.x; dst[t][1] = a.y; dst[t][2] = b.x; dst[t][3] = b.y;
  }
}
// Rows >= valid are not written.
template <int NTL>
__device__ __forceinline__ void frag_st(const float (&src)[NTL][4], float *M, size_t ld, int r0, int c0,
                                        int lane, int valid) {
  const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int t = 0; t < NTL; ++t) {
    if (r0 + gid < valid)
      *reinterpret_cast<float2 *>(M + (size_t)(r0 + gid) * ld + c0 + 8 * t + 2 * tig) = make_float2(src[t][0], src[t][1]);
    if (r0 + gid + 8 < valid)
      *reinterpret_cast<float2 *>(M + (size_t)(r0 + gid + 8) * ld + c0 + 8 * t + 2 * tig) = make_float2(src[t][2], src[t][3]);
  }
}

// Sum of the two rows (gid, gid + 8) a lane holds over the warp's columns:
// returned in every lane of the quad.
template <int NTL, class F>
__device__ __forceinline__ void quad_row_sums(float (&acc)[NTL][4], F weight, int r0, int c0,
                                              int lane, float &s_lo, float &s_hi) {
  const int gid = lane >> 2, tig = lane & 3;
  float a = 0.f, b = 0.f;
#pragma unroll
  for (int t = 0; t < NTL; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = r0 + gid + 8 * (e >> 1), c = c0 + 8 * t + 2 * tig + (e & 1);
      const float x = acc[t][e] * weight(r, c);
      if (e < 2) a += x; else b += x;
    }
  a += __shfl_xor_sync(0xffffffffu, a, 1);
  a += __shfl_xor_sync(0xffffffffu, a, 2);
  b += __shfl_xor_sync(0xffffffffu, b, 1);
  b += __shfl_xor_sync(0xffffffffu, b, 2);
  s_lo = a;
  s_hi = b;
}

// ---- asynchronous tile copies -----------------------------------------------
// 16 bytes global -> shared, or 16 zero bytes when !ok (the source is then
// not read).
__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool ok) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(sm100::smem_addr(dst)),
               "l"(src), "r"(ok ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}
// dst[r][0..COLS) (row stride ld elements) <- src[r * stride + 0..COLS) for r
// < valid, zeros for valid <= r < ROWS.  Rows of dst and src 16-byte aligned.
template <int ROWS, int COLS, int NTH = NT, typename E>
__device__ __forceinline__ void tile_async(E *dst, int ld, const E *src, size_t stride, int valid,
                                           int tid) {
  constexpr int PER = 16 / sizeof(E), V = COLS / PER;
  for (int x = tid; x < ROWS * V; x += NTH) {
    const int r = x / V, c = PER * (x - r * V);
    const bool ok = r < valid;
    cp_async16(dst + r * ld + c, ok ? src + (size_t)r * stride + c : src, ok);
  }
}
// dst[r * stride + c] = src[r][c] (row stride ld) for r < ROWS, c < COLS.
template <int ROWS, int COLS, int NTH = NT>
__device__ __forceinline__ void store_tile(float *dst, size_t stride, const float *src, int ld,
                                           int tid) {
  constexpr int V4 = COLS / 4;
  for (int x = tid; x < ROWS * V4; x += NTH) {
    const int r = x / V4, c = 4 * (x - r * V4);
    *reinterpret_cast<float4 *>(dst + (size_t)r * stride + c) =
        *reinterpret_cast<const float4 *>(src + r * ld + c);
  }
}
template <int ROWS, int COLS, int NTH = NT>
__device__ __forceinline__ void zero_tile(float *dst, int ld, int tid) {
  for (int x = tid; x < ROWS * COLS; x += NTH) dst[(x / COLS) * ld + x % COLS] = 0.f;
}

// Row stride (elements) of an input tile kept in its own type in shared
// memory: conflict-free for the fragment reads of mma3_rows in both
// orientations.
template <typename E>
constexpr int in_ld(int D) { return sizeof(E) == 2 ? D + 8 : D + 4; }
constexpr size_t up16(size_t x) { return (x + 15) & ~(size_t)15; }

struct ChunkPos {
  int n, start, len;
};
// Sequence, first token and length of global chunk c; false past the last chunk.
__device__ __forceinline__ bool chunk_pos(const Params &p, int c, ChunkPos &cp) {
  if (c >= p.ph->total_chunks) return false;
  const int kk = tp::owner_of_chunk(p.ne_cs, p.ph->n_nonempty, c);
  const int n = p.ne_seq[kk];
  cp.n = n;
  cp.start = p.cu[n] + C * (c - p.ne_cs[kk]);
  cp.len = min(C, p.cu[n + 1] - cp.start);
  return true;
}

// ---- prep: P, E . K K^T, Tm, W, U~ and G of one (chunk, value head) ----------
template <typename TI, int DK, int DV>
struct PrepSmem {
  static constexpr int LQ = in_ld<TI>(DK), LV = in_ld<TI>(DV);
  static constexpr size_t OQ = 0, OK = OQ + up16(C * LQ * sizeof(TI)), OV = OK + up16(C * LQ * sizeof(TI)),
                          OA = OV + up16(C * LV * sizeof(TI)), OT = OA + C * LD64 * 4,
                          OY = OT + C * LD64 * 4, OG = OY + up16(3 * 16 * 17 * 4), OB = OG + C * 8,
                          OBG = OB + C * 4, BYTES = OBG + C * 4;
};

template <typename TI, int DK, int DV>
__global__ void __launch_bounds__(NT) prep_kernel(const Params p) {
  using L = PrepSmem<TI, DK, DV>;
  extern __shared__ __align__(16) unsigned char smb[];
  TI *Qs = reinterpret_cast<TI *>(smb + L::OQ), *Ks = reinterpret_cast<TI *>(smb + L::OK),
     *Vs = reinterpret_cast<TI *>(smb + L::OV);
  float *As = reinterpret_cast<float *>(smb + L::OA), *Ts = reinterpret_cast<float *>(smb + L::OT),
        *Ysc = reinterpret_cast<float *>(smb + L::OY), *sB = reinterpret_cast<float *>(smb + L::OB),
        *sBG = reinterpret_cast<float *>(smb + L::OBG);
  double *sG = reinterpret_cast<double *>(smb + L::OG);
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  ChunkPos cp;
  if (!chunk_pos(p, blockIdx.x, cp)) return;
  const int h = blockIdx.y, hk = h / (p.Hv / p.Hqk);
  const size_t u = (size_t)blockIdx.x * p.Hv + h;
  const TI *q = static_cast<const TI *>(p.q), *k = static_cast<const TI *>(p.k),
           *v = static_cast<const TI *>(p.v);
  const size_t qoff = ((size_t)cp.start * p.Hqk + hk) * DK, qstride = (size_t)p.Hqk * DK;
  tile_async<C, DK>(Qs, L::LQ, q + qoff, qstride, cp.len, tid);
  tile_async<C, DK>(Ks, L::LQ, k + qoff, qstride, cp.len, tid);
  tile_async<C, DV>(Vs, L::LV, v + ((size_t)cp.start * p.Hv + h) * DV, (size_t)p.Hv * DV, cp.len, tid);
  cp_commit();
  zero_tile<C, C>(Ts, LD64, tid);
  if (w == 0) {  // prefix sums of the clamped log-decays, in fp64 (2 tokens per lane)
    const int t0 = 2 * lane;
    float g0 = 0.f, g1 = 0.f, b0 = 0.f, b1 = 0.f;
    if (t0 < cp.len) { g0 = fmaxf(p.g[(size_t)(cp.start + t0) * p.Hv + h], kGmin); b0 = p.beta[(size_t)(cp.start + t0) * p.Hv + h]; }
    if (t0 + 1 < cp.len) { g1 = fmaxf(p.g[(size_t)(cp.start + t0 + 1) * p.Hv + h], kGmin); b1 = p.beta[(size_t)(cp.start + t0 + 1) * p.Hv + h]; }
    double s = (double)g0 + (double)g1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const double x = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += x;
    }
    const double G1 = s, G0 = s - g1;
    sG[t0] = G0; sG[t0 + 1] = G1;
    sB[t0] = b0; sB[t0 + 1] = b1;
    sBG[t0] = b0 * expf((float)G0); sBG[t0 + 1] = b1 * expf((float)G1);
    p.G[u * C + t0] = G0;
    p.G[u * C + t0 + 1] = G1;
  }
  cp_wait<0>();
  __syncthreads();
  {  // QK^T and KK^T: warp rows 16 (w & 3), columns 32 (w >> 2)
    const int r0 = 16 * (w & 3), c0 = 32 * (w >> 2);
    float aq[4][4], ak[4][4];
    zero_acc(aq);
    zero_acc(ak);
    constexpr bool EX = sizeof(TI) == 2;  // raw bf16 inputs are exact bf16 operands
    mma3_rows<DK, 4, EX, EX>(aq, [&](int r, int c) { return to_f32(Qs[(r0 + r) * L::LQ + c]); },
                      [&](int r, int c) { return to_f32(Ks[(c0 + c) * L::LQ + r]); }, lane);
    mma3_rows<DK, 4, EX, EX>(ak, [&](int r, int c) { return to_f32(Ks[(r0 + r) * L::LQ + c]); },
                      [&](int r, int c) { return to_f32(Ks[(c0 + c) * L::LQ + r]); }, lane);
    float *P = p.P + u * C * C, *EKK = p.EKK + u * C * C;
    const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int i = r0 + gid + 8 * hr, j = c0 + 8 * t + 2 * tig;
        float pv[2], ev[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float E = (i >= j + e) ? expf((float)(sG[i] - sG[j + e])) : 0.f;
          pv[e] = (i >= j + e) ? E * aq[t][2 * hr + e] : 0.f;
          ev[e] = (i > j + e) ? E * ak[t][2 * hr + e] : 0.f;
          As[i * LD64 + j + e] = sB[i] * ev[e];
        }
        *reinterpret_cast<float2 *>(P + i * C + j) = make_float2(pv[0], pv[1]);
        *reinterpret_cast<float2 *>(EKK + i * C + j) = make_float2(ev[0], ev[1]);
      }
  }
  __syncthreads();
  chunk::ut_solve<NT, 1>(As, Ts, Ysc, tid);  // ends with a barrier of all NT threads
  store_tile<C, C>(p.Tm + u * C * C, C, Ts, LD64, tid);
  {  // W = Tm diag(beta gamma) K and U~ = Tm diag(beta) V: rows 16 (w & 3), column halves
    const int r0 = 16 * (w & 3);
    {
      const int c0 = (w >> 2) * (DK / 2);
      float acc[DK / 16][4];
      zero_acc(acc);
      mma3_rows<C, DK / 16, false, sizeof(TI) == 2>(
          acc, [&](int r, int c) { return Ts[(r0 + r) * LD64 + c] * sBG[c]; },
          [&](int r, int c) { return to_f32(Ks[r * L::LQ + c0 + c]); }, lane);
      frag_st(acc, p.W + u * C * DK, DK, r0, c0, lane, C);
    }
    {
      const int c0 = (w >> 2) * (DV / 2);
      float acc[DV / 16][4];
      zero_acc(acc);
      mma3_rows<C, DV / 16, false, sizeof(TI) == 2>(
          acc, [&](int r, int c) { return Ts[(r0 + r) * LD64 + c] * sB[c]; },
          [&](int r, int c) { return to_f32(Vs[r * L::LV + c0 + c]); }, lane);
      frag_st(acc, p.Ut + u * C * DV, DV, r0, c0, lane, C);
    }
  }
}

// ---- forward chain: S0 and U of every chunk, a whole head (Dv state rows) ----
// With bf16 inputs the K, U~ and G tiles are double-buffered: chunk j + 1's
// are in flight while chunk j computes (fp32 inputs do not fit twice).
template <typename TI, int DK, int DV>
struct FwdSmem {
  static constexpr int NB = sizeof(TI) == 2 ? 2 : 1;
  static constexpr int LS = DK + 4, LW = DK + 4, LK = in_ld<TI>(DK), LU = DV + 8;
  static constexpr size_t KB = up16(C * LK * sizeof(TI)), UB = C * LU * 4;
  static constexpr size_t OS = 0, OW = OS + DV * LS * 4, OK = OW + C * LW * 4, OU = OK + NB * KB,
                          OG = OU + NB * UB, OKD = OG + NB * C * 8, BYTES = OKD + C * 4;
};

// One CTA of NTR threads per (non-empty sequence kk, value head h).
template <typename TI, int DK, int DV>
__device__ __forceinline__ void fwd_chain_body(const Params &p, unsigned char *smb, int kk, int h) {
  using L = FwdSmem<TI, DK, DV>;
  constexpr int NB = L::NB;
  constexpr int NW = NTR / 32;               // 16 warps
  constexpr int RG = DV / 16, CG = NW / RG;  // state update: row groups x column groups
  float *S = reinterpret_cast<float *>(smb + L::OS), *Ws = reinterpret_cast<float *>(smb + L::OW),
        *sKd = reinterpret_cast<float *>(smb + L::OKD);
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (kk >= p.ph->n_nonempty) return;
  const int n = p.ne_seq[kk], c0 = p.ne_cs[kk], nch = p.ne_cs[kk + 1] - c0;
  const int cs = p.cu[n], Lseq = p.cu[n + 1] - cs;
  const int hk = h / (p.Hv / p.Hqk);
  const TI *k = static_cast<const TI *>(p.k);
  const size_t srow = ((size_t)n * p.Hv + h) * DV;  // first state row of the head
  auto Kb = [&](int j) { return reinterpret_cast<TI *>(smb + L::OK + (j % NB) * L::KB); };
  auto Ub = [&](int j) { return reinterpret_cast<float *>(smb + L::OU + (j % NB) * L::UB); };
  auto Gb = [&](int j) { return reinterpret_cast<double *>(smb + L::OG + (j % NB) * C * 8); };
  auto issue_tiles = [&](int j) {  // K, U~ and G of chunk j, one commit group
    const size_t u = (size_t)(c0 + j) * p.Hv + h;
    const int start = cs + C * j, len = min(C, Lseq - C * j);
    tile_async<C, DK, NTR>(Kb(j), L::LK, k + ((size_t)start * p.Hqk + hk) * DK, (size_t)p.Hqk * DK, len, tid);
    tile_async<C, DV, NTR>(Ub(j), L::LU, p.Ut + u * C * DV, DV, C, tid);
    tile_async<1, C, NTR>(Gb(j), C, p.G + u * C, 0, 1, tid);
    cp_commit();
  };
  if (p.s0) tile_async<DV, DK, NTR>(S, L::LS, p.s0 + srow * DK, DK, DV, tid);
  else zero_tile<DV, DK, NTR>(S, L::LS, tid);
  tile_async<C, DK, NTR>(Ws, L::LW, p.W + ((size_t)c0 * p.Hv + h) * C * DK, DK, C, tid);
  issue_tiles(0);  // S0, the first W and chunk 0's tiles in one group
  for (int j = 0; j < nch; ++j) {
    const size_t u = (size_t)(c0 + j) * p.Hv + h;
    const int len = min(C, Lseq - C * j);
    if (NB == 2 && j + 1 < nch) {
      issue_tiles(j + 1);  // into the buffers chunk j - 1 used
      cp_wait<1>();
    } else {
      if (NB == 1 && j > 0) issue_tiles(j);
      cp_wait<0>();
    }
    __syncthreads();
    TI *Ks = Kb(j);
    float *Us = Ub(j);
    const double *sG = Gb(j);
    store_tile<DV, DK, NTR>(p.S0 + u * DV * DK, DK, S, L::LS, tid);
    if (tid < C) sKd[tid] = tid < len ? expf((float)(sG[len - 1] - sG[tid])) : 0.f;
    {  // U = U~ - W S^T: token rows 16 (w & 3), state rows DV / 4 (w >> 2)
      const int r0 = 16 * (w & 3), vb = (w >> 2) * (DV / 4);
      float acc[DV / 32][4];
      zero_acc(acc);
      mma3_rows<DK>(acc, [&](int r, int c) { return Ws[(r0 + r) * L::LW + c]; },
                    [&](int r, int c) { return S[(vb + c) * L::LS + r]; }, lane);
      for_frag(acc, r0, vb, lane, [&](int i, int c, float &x) {
        x = Us[i * L::LU + c] - x;
        Us[i * L::LU + c] = x;
      });
      frag_st(acc, p.U + u * C * DV, DV, r0, vb, lane, C);
    }
    __syncthreads();
    if (j + 1 < nch) {
      tile_async<C, DK, NTR>(Ws, L::LW, p.W + (u + p.Hv) * C * DK, DK, C, tid);  // next chunk's W
      cp_commit();
      // S <- gamma_C S + U^T diag(kdec) K: state rows 16 (w % RG), columns DK / CG (w / RG)
      const float gC = expf((float)sG[len - 1]);
      const int r0 = 16 * (w % RG), kb = (w / RG) * (DK / CG);
      float acc[DK / CG / 8][4];
      for_frag(acc, r0, kb, lane, [&](int r, int c, float &x) { x = gC * S[r * L::LS + c]; });
      mma3_rows<C, DK / CG / 8, false, sizeof(TI) == 2>(
          acc, [&](int r, int c) { return Us[c * L::LU + r0 + r] * sKd[c]; },
          [&](int r, int c) { return to_f32(Ks[r * L::LK + kb + c]); }, lane);
      for_frag(acc, r0, kb, lane, [&](int r, int c, float &x) { S[r * L::LS + c] = x; });
      __syncthreads();
    }
  }
}

// ---- reverse chain: dS1 and dU of every chunk, last to first ------------------
// P and K are fetched one chunk ahead into single buffers (the dU product is
// their only reader).  With bf16 inputs dO, Q, W and G are double-buffered:
// chunk j - 1's are in flight while chunk j computes.
template <typename TI, int DK, int DV>
struct RevSmem {
  static constexpr int NB = sizeof(TI) == 2 ? 2 : 1;
  static constexpr int LS = DK + 4, LK = in_ld<TI>(DK), LW = DK + 8, LO = SL + 8;
  static constexpr size_t KB = up16(C * LK * sizeof(TI)), OB = C * LO * 4, WB = C * LW * 4;
  static constexpr size_t OS = 0, OP = OS + SL * LS * 4, OK = OP + C * LD64 * 4, OU = OK + KB,
                          OO = OU + OB, OQ = OO + NB * OB, OW = OQ + NB * KB, OG = OW + NB * WB,
                          OGM = OG + NB * C * 8, BYTES = OGM + C * 4;
  static_assert(BYTES <= 232448, "reverse chain above the 227 KB of shared memory a CTA may use");
};

// One CTA of NTR threads per (non-empty sequence kk, value head h, SL state
// rows from v0).
template <typename TI, int DK, int DV>
__device__ __forceinline__ void rev_chain_body(const Params &p, unsigned char *smb, int kk, int h, int v0) {
  using L = RevSmem<TI, DK, DV>;
  constexpr int NB = L::NB;
  float *dS = reinterpret_cast<float *>(smb + L::OS), *Ps = reinterpret_cast<float *>(smb + L::OP),
        *dUs = reinterpret_cast<float *>(smb + L::OU), *sGm = reinterpret_cast<float *>(smb + L::OGM);
  TI *Ks = reinterpret_cast<TI *>(smb + L::OK);
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int gid = lane >> 2;
  if (kk >= p.ph->n_nonempty) return;
  const int n = p.ne_seq[kk], c0 = p.ne_cs[kk], nch = p.ne_cs[kk + 1] - c0;
  const int cs = p.cu[n], Lseq = p.cu[n + 1] - cs;
  const int hk = h / (p.Hv / p.Hqk);
  const TI *q = static_cast<const TI *>(p.q), *k = static_cast<const TI *>(p.k);
  const size_t srow = ((size_t)n * p.Hv + h) * DV + v0;
  const size_t qstride = (size_t)p.Hqk * DK;
  const float scale = p.scale;
  auto Ob = [&](int j) { return reinterpret_cast<float *>(smb + L::OO + (j % NB) * L::OB); };
  auto Qb = [&](int j) { return reinterpret_cast<TI *>(smb + L::OQ + (j % NB) * L::KB); };
  auto Wb = [&](int j) { return reinterpret_cast<float *>(smb + L::OW + (j % NB) * L::WB); };
  auto Gb = [&](int j) { return reinterpret_cast<double *>(smb + L::OG + (j % NB) * C * 8); };
  auto issue_tiles = [&](int j) {  // dO, Q, W and G of chunk j, one commit group
    const size_t u = (size_t)(c0 + j) * p.Hv + h;
    const int start = cs + C * j, len = min(C, Lseq - C * j);
    tile_async<C, SL, NTR>(Ob(j), L::LO, p.dO + ((size_t)start * p.Hv + h) * DV + v0, (size_t)p.Hv * DV, len, tid);
    tile_async<C, DK, NTR>(Qb(j), L::LK, q + ((size_t)start * p.Hqk + hk) * DK, qstride, len, tid);
    tile_async<C, DK, NTR>(Wb(j), L::LW, p.W + u * C * DK, DK, C, tid);
    tile_async<1, C, NTR>(Gb(j), C, p.G + u * C, 0, 1, tid);
    cp_commit();
  };
  if (p.dSf) tile_async<SL, DK, NTR>(dS, L::LS, p.dSf + srow * DK, DK, SL, tid);
  else zero_tile<SL, DK, NTR>(dS, L::LS, tid);
  {  // P and K of the last chunk (later ones are fetched one chunk ahead)
    const size_t u = (size_t)(c0 + nch - 1) * p.Hv + h;
    const int start = cs + C * (nch - 1), len = min(C, Lseq - C * (nch - 1));
    tile_async<C, C, NTR>(Ps, LD64, p.P + u * C * C, C, C, tid);
    tile_async<C, DK, NTR>(Ks, L::LK, k + ((size_t)start * p.Hqk + hk) * DK, qstride, len, tid);
  }
  issue_tiles(nch - 1);  // the final-state gradient, the last P, K and tiles in one group
  const int r0 = 16 * (w & 3);
  for (int j = nch - 1; j >= 0; --j) {
    const size_t u = (size_t)(c0 + j) * p.Hv + h;
    const int start = cs + C * j, len = min(C, Lseq - C * j);
    if (NB == 2 && j > 0) {
      issue_tiles(j - 1);  // into the buffers chunk j + 1 used
      cp_wait<1>();
    } else {
      if (NB == 1 && j < nch - 1) issue_tiles(j);
      cp_wait<0>();
    }
    __syncthreads();
    const float *dOs = Ob(j), *Ws = Wb(j);
    const TI *Qs = Qb(j);
    const double *sG = Gb(j);
    store_tile<SL, DK, NTR>(p.dS1 + (u * DV + v0) * DK, DK, dS, L::LS, tid);
    if (tid < C) sGm[tid] = tid < len ? expf((float)sG[tid]) : 0.f;
    {  // dU = P^T dO' + diag(kdec) K dS^T: token rows 16 (w & 3), state rows 16 (w >> 2)
      const int vb = 16 * (w >> 2);
      float a1[2][4], a2[2][4];
      zero_acc(a1);
      zero_acc(a2);
      mma3_rows<C>(a1, [&](int r, int c) { return Ps[c * LD64 + r0 + r]; },
                       [&](int r, int c) { return dOs[r * L::LO + vb + c]; }, lane);
      mma3_rows<DK, 2, sizeof(TI) == 2, false>(a2, [&](int r, int c) { return to_f32(Ks[(r0 + r) * L::LK + c]); },
                        [&](int r, int c) { return dS[(vb + c) * L::LS + r]; }, lane);
      const double Gl = sG[len - 1];
      const int i0 = r0 + gid, i1 = i0 + 8;
      const float kd0 = i0 < len ? expf((float)(Gl - sG[i0])) : 0.f;
      const float kd1 = i1 < len ? expf((float)(Gl - sG[i1])) : 0.f;
      const int tig = lane & 3;
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = r0 + gid + 8 * (e >> 1), c = vb + 8 * t + 2 * tig + (e & 1);
          a1[t][e] = scale * a1[t][e] + (e < 2 ? kd0 : kd1) * a2[t][e];
          dUs[i * L::LO + c] = a1[t][e];
        }
      frag_st(a1, p.dU + u * C * DV + v0, DV, r0, vb, lane, C);
    }
    __syncthreads();
    if (j > 0) {  // the previous chunk's P and K into the freed buffers
      const size_t up = u - p.Hv;
      const int sp = start - C;
      tile_async<C, C, NTR>(Ps, LD64, p.P + up * C * C, C, C, tid);
      tile_async<C, DK, NTR>(Ks, L::LK, k + ((size_t)sp * p.Hqk + hk) * DK, qstride, C, tid);
      cp_commit();
    }
    {  // dS <- gamma_C dS + dO'^T diag(gamma) Q - dU^T W: state rows 16 (w & 3), columns DK / 4 (w >> 2)
      const float gC = expf((float)sG[len - 1]);
      const int kb = (w >> 2) * (DK / 4);
      float acc[DK / 32][4];
      for_frag(acc, r0, kb, lane, [&](int r, int c, float &x) { x = gC * dS[r * L::LS + c]; });
      mma3_rows<C, DK / 32, false, sizeof(TI) == 2>(acc, [&](int r, int c) { return scale * dOs[c * L::LO + r0 + r] * sGm[c]; },
                       [&](int r, int c) { return to_f32(Qs[r * L::LK + kb + c]); }, lane);
      mma3_rows<C>(acc, [&](int r, int c) { return -dUs[c * L::LO + r0 + r]; },
                       [&](int r, int c) { return Ws[r * L::LW + kb + c]; }, lane);
      for_frag(acc, r0, kb, lane, [&](int r, int c, float &x) { dS[r * L::LS + c] = x; });
    }
    __syncthreads();
  }
  if (p.ds0) store_tile<SL, DK, NTR>(p.ds0 + srow * DK, DK, dS, L::LS, tid);
}

// ---- both chains in one launch ----------------------------------------------
// The two chains do not depend on each other.  CTAs [0, N Hv Dv / SL) run the
// reverse chain (SL rows each), the next N Hv the forward chain (a whole head
// each); CTAs start in index order, so at 48 heads all 144 share one wave, one
// per SM, whatever the scheduler does with separate launches.
template <typename TI, int DK, int DV>
struct ChainSmem {
  static constexpr size_t F = FwdSmem<TI, DK, DV>::BYTES, R = RevSmem<TI, DK, DV>::BYTES;
  static constexpr size_t BYTES = F > R ? F : R;
};

template <typename TI, int DK, int DV>
__global__ void __launch_bounds__(NTR, 1) chains_kernel(const Params p) {
  extern __shared__ __align__(16) unsigned char smb[];
  constexpr int R = DV / SL;
  const int nrev = p.N * p.Hv * R;
  int b = blockIdx.x;
  if (b < nrev) {
    const int kk = b / (p.Hv * R), rem = b - kk * (p.Hv * R);
    rev_chain_body<TI, DK, DV>(p, smb, kk, rem / R, SL * (rem % R));
  } else {
    b -= nrev;
    fwd_chain_body<TI, DK, DV>(p, smb, b / p.Hv, b % p.Hv);
  }
}

// ---- tcgen05 building blocks -----------------------------------------------
// Operands of the 5th-generation tensor-core products are bf16 images in
// shared memory, 128-byte swizzled, each fp32 value split into hi =
// bf16(x) and lo = bf16(x - hi) (both rounded to nearest, |x - hi - lo| <=
// 2^-18 |x|); a product is hi*hi' + hi*lo' + lo*hi' (3 MMAs per K step,
// about 2^-16 relative), accumulated in fp32 in tensor memory.
//   K-major image of an R x K operand (R = 128 rows): K blocks of 64 columns,
//   R x 128 bytes each; element (r, k) at block k / 64, sw128_off(r, (k % 64) / 8).
//   MN-major image of a K x N operand: N blocks of 64 columns, K x 128 bytes
//   each; element (k, n) at block n / 64, sw128_off(k, (n % 64) / 8).
// Both store 8 consecutive elements of a row as one 16-byte chunk.
__device__ __forceinline__ void split8_bf16(const float *x, uint4 &hi, uint4 &lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat162 hb = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
    const float2 hf = __bfloat1622float2(hb);
    const __nv_bfloat162 lb = __floats2bfloat162_rn(x[2 * e] - hf.x, x[2 * e + 1] - hf.y);
    h[e] = *reinterpret_cast<const uint32_t *>(&hb);
    l[e] = *reinterpret_cast<const uint32_t *>(&lb);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}
// Store the split of x[0..8) as chunk `chunk` of row `row` of the images
// whose blocks start at hi_base / lo_base (block already selected).
__device__ __forceinline__ void st_img8(unsigned char *hi_base, unsigned char *lo_base, int row,
                                        int chunk, const float *x) {
  uint4 h, l;
  split8_bf16(x, h, l);
  const uint32_t off = sm100::sw128_off((uint32_t)row, (uint32_t)chunk);
  *reinterpret_cast<uint4 *>(hi_base + off) = h;
  *reinterpret_cast<uint4 *>(lo_base + off) = l;
}
// 8 consecutive fp32 values from global memory (16-byte aligned), or zeros.
__device__ __forceinline__ void ld8(const float *src, bool ok, float *x) {
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
  if (ok) {
    a = *reinterpret_cast<const float4 *>(src);
    b = *reinterpret_cast<const float4 *>(src + 4);
  }
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
// 32 consecutive input elements (16-byte aligned) as fp32, by 16-byte loads.
__device__ __forceinline__ void ld32(const float *src, float *x) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 a = *reinterpret_cast<const float4 *>(src + 4 * i);
    x[4 * i] = a.x; x[4 * i + 1] = a.y; x[4 * i + 2] = a.z; x[4 * i + 3] = a.w;
  }
}
__device__ __forceinline__ void ld32(const __nv_bfloat16 *src, float *x) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 a = *reinterpret_cast<const uint4 *>(src + 8 * i);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[8 * i + 2 * e] = __uint_as_float(w[e] << 16);
      x[8 * i + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
  }
}

// 3-term product D (+)= A B over KSTEPS K steps of 16, A K-major (blocks of
// 64 K at a_blk bytes), B MN-major (K rows of 128 bytes, N blocks at b_lbo).
// Issued by one thread.
template <int KSTEPS>
__device__ __forceinline__ void umma3_kmaj_mn(uint32_t d_tmem, uint32_t a_hi, uint32_t a_lo,
                                              uint32_t a_blk, uint32_t b_hi, uint32_t b_lo,
                                              uint32_t b_lbo, uint32_t idesc, bool accumulate) {
#pragma unroll
  for (int ks = 0; ks < KSTEPS; ++ks) {
    const uint32_t ao = (ks >> 2) * a_blk + (ks & 3) * 32, bo = ks * 2048;
    const uint64_t ah = sm100::sdesc_sw128(a_hi + ao, 16, 1024), al = sm100::sdesc_sw128(a_lo + ao, 16, 1024);
    const uint64_t bh = sm100::sdesc_sw128(b_hi + bo, b_lbo, 1024), bl = sm100::sdesc_sw128(b_lo + bo, b_lbo, 1024);
    sm100::mma_bf16(d_tmem, al, bh, idesc, (accumulate || ks > 0) ? 1u : 0u);
    sm100::mma_bf16(d_tmem, ah, bl, idesc, 1u);
    sm100::mma_bf16(d_tmem, ah, bh, idesc, 1u);
  }
}
// Every thread waits for an mbarrier phase (bounded); false when it gave up,
// which is recorded in the status word.  No thread leaves early, so the
// CTA-wide barriers that follow are reached by all.
__device__ __forceinline__ bool cta_wait(uint32_t bar, uint32_t parity, volatile int *ctl, int32_t *status) {
  if (sm100::mbar_wait(bar, parity, ctl)) {
    sm100::tc_fence_after();
    return true;
  }
  ctl[0] = 1;
  report_status(status, GDN_ERR_DEVICE_TIMEOUT);
  return false;
}

// ---- products with S0 and dS1 of one (chunk, value head), on tcgen05 ----------
// D1 = [dO; dU] S0 (M = 128: rows 0-63 the chunk's dO, rows 64-127 its dU) and
// D2 = U dS1 (rows 0-63; rows 64-127 of that A image hold stale rows and are
// not read), both N = Dk, K = Dv, accumulators in tensor memory:
//   dQ part  diag(scale gamma) (dO S0),  dgamma_t = scale q_t . (dO S0)_t
//   dW       -(dU S0)
//   dK part  diag(kdec) (U dS1),         dkdec_t = k_t . (U dS1)_t
//   dgamma_C = <dS1, S0>
// K runs in halves of 64 (one operand image each), so a CTA holds 64 KB of
// images and two CTAs share an SM (and its 512 TMEM columns): one's loads run
// beside the other's products and epilogue.  Order at Dv = 128: D1 half 0,
// D2 half 0, D2 half 1, D1 half 1; each B image is read back for <dS1, S0>
// by the step that overwrites it with its partner (S0 half 0 by dS1 half 0,
// dS1 half 1 by S0 half 1).  One thread issues the MMAs; all threads build
// the images and read the results (warp w: TMEM lanes 32 (w % 4) .. + 31).
template <int DK, int DV>
struct StateGradSmem {
  static constexpr int NKH = DV / 64;                     // K halves
  static constexpr uint32_t A_BYTES = 128 * 128;          // 128 rows x 64 K, K-major
  static constexpr uint32_t B_LBO = 64 * 128;             // one 64-column N block of 64 K rows, MN-major
  static constexpr uint32_t B_BYTES = (DK / 64) * B_LBO;
  static constexpr uint32_t OAH = 0, OAL = A_BYTES, OBH = 2 * A_BYTES, OBL = OBH + B_BYTES,
                            OG = OBL + B_BYTES, ORED = OG + C * 8, OBAR = ORED + (4 * C + 8) * 4,
                            OMISC = OBAR + 16, USED = OMISC + 32;
  // at least 78 KB: no third CTA on an SM whose TMEM two of them fill
  static constexpr uint32_t BYTES = USED > 78 * 1024 ? USED : 78 * 1024;
  static constexpr uint32_t TMEM_COLS = 2 * DK;  // 128 or 256
};

// Rows of 8-element chunks, NT threads, N items each: item it of thread tid is
// chunk (tid + NT it) % CPR of row (tid + NT it) / CPR.
template <int CPR>
__device__ __forceinline__ void item_pos(int tid, int it, int &r, int &c) {
  const int idx = tid + NT * it;
  r = idx / CPR;
  c = idx % CPR;
}
// Store x (rows of 64 K columns) into the A image (K-major, one K block).
template <int N>
__device__ __forceinline__ void st_a_items(unsigned char *AH, unsigned char *AL, const float (&x)[N][8], int tid) {
#pragma unroll
  for (int it = 0; it < N; ++it) {
    int r, c;
    item_pos<8>(tid, it, r, c);
    st_img8(AH, AL, r, c, x[it]);
  }
}
// Store x (64 K rows x DK, MN-major) into the B image; with DOT, first add
// <old image, x> to dot (the old value rebuilt as hi + lo).
template <int N, int DK, bool DOT>
__device__ __forceinline__ void st_b_items(unsigned char *BH, unsigned char *BL, uint32_t lbo, const float (&x)[N][8],
                                           int tid, float &dot) {
#pragma unroll
  for (int it = 0; it < N; ++it) {
    int v, c;
    item_pos<DK / 8>(tid, it, v, c);
    const uint32_t off = sm100::sw128_off((uint32_t)v, (uint32_t)(c & 7)) + (c >> 3) * lbo;
    if (DOT) {
      const uint4 hv = *reinterpret_cast<const uint4 *>(BH + off), lv = *reinterpret_cast<const uint4 *>(BL + off);
      const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w}, lw[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float o0 = __uint_as_float(hw[e] << 16) + __uint_as_float(lw[e] << 16);
        const float o1 = __uint_as_float(hw[e] & 0xffff0000u) + __uint_as_float(lw[e] & 0xffff0000u);
        dot = fmaf(x[it][2 * e], o0, fmaf(x[it][2 * e + 1], o1, dot));
      }
    }
    uint4 hi, lo;
    split8_bf16(x[it], hi, lo);
    *reinterpret_cast<uint4 *>(BH + off) = hi;
    *reinterpret_cast<uint4 *>(BL + off) = lo;
  }
}

template <typename TI, int DK, int DV>
__global__ void __launch_bounds__(NT, 2) grads_state_kernel(const Params p) {
  using L = StateGradSmem<DK, DV>;
  constexpr int NKH = L::NKH;
  constexpr int AI = 128 * 8 / NT, UI = C * 8 / NT, BI = 64 * (DK / 8) / NT;  // items per thread
  extern __shared__ __align__(1024) unsigned char smb[];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  ChunkPos cp;
  if (!chunk_pos(p, blockIdx.x, cp)) return;
  const uint32_t sb = sm100::smem_addr(smb);
  if (sb & 1023u) {  // swizzled operand images need 1024-byte alignment
    if (tid == 0) report_status(p.status, GDN_ERR_UNSUPPORTED);
    return;
  }
  const int h = blockIdx.y, hk = h / (p.Hv / p.Hqk);
  const size_t u = (size_t)blockIdx.x * p.Hv + h;
  const int len = cp.len;
  volatile int *ctl = reinterpret_cast<volatile int *>(smb + L::OMISC + 4);
  const uint32_t bar_mma = sb + L::OBAR, bar_drain = sb + L::OBAR + 8;
  double *sG = reinterpret_cast<double *>(smb + L::OG);
  float *red = reinterpret_cast<float *>(smb + L::ORED);
  unsigned char *AH = smb + L::OAH, *AL = smb + L::OAL, *BH = smb + L::OBH, *BL = smb + L::OBL;
  if (tid == 0) {
    sm100::mbar_init(bar_mma, 1);
    sm100::mbar_init(bar_drain, 1);
    ctl[0] = 0;
    ctl[1] = (int)header_wait_limit_us(p.status);
    sm100::fence_barrier_init();
  }
  if (w == 0) {
    sm100::tmem_alloc(sb + L::OMISC, L::TMEM_COLS);
    sm100::tmem_relinquish();
  }
  if (tid < C) sG[tid] = p.G[u * C + tid];
  const float *S0g = p.S0 + u * DV * DK, *S1g = p.dS1 + u * DV * DK, *Uc = p.U + u * C * DV;
  const float *dOc = p.dO + ((size_t)cp.start * p.Hv + h) * DV, *dUc = p.dU + u * C * DV;
  const size_t dOs = (size_t)p.Hv * DV;
  // loads of one K half (value columns [64 kh, + 64)) into registers
  auto ld_dodu = [&](int kh, float (&x)[AI][8]) {
#pragma unroll
    for (int it = 0; it < AI; ++it) {
      int r, c;
      item_pos<8>(tid, it, r, c);
      const int col = 64 * kh + 8 * c;
      ld8(r < C ? dOc + (size_t)r * dOs + col : dUc + (size_t)(r - C) * DV + col, r >= C || r < len, x[it]);
    }
  };
  auto ld_u = [&](int kh, float (&x)[UI][8]) {
#pragma unroll
    for (int it = 0; it < UI; ++it) {
      int r, c;
      item_pos<8>(tid, it, r, c);
      ld8(Uc + (size_t)r * DV + 64 * kh + 8 * c, true, x[it]);
    }
  };
  auto ld_state = [&](const float *Sg, int kh, float (&x)[BI][8]) {
#pragma unroll
    for (int it = 0; it < BI; ++it) {
      int v, c;
      item_pos<DK / 8>(tid, it, v, c);
      ld8(Sg + (size_t)(64 * kh + v) * DK + 8 * c, true, x[it]);
    }
  };
  constexpr uint32_t IDESC = sm100::idesc_bf16(128, DK, 0, 1);
  uint32_t tmem = 0;
  // images written -> visible to the tensor cores -> one thread issues
  auto issue = [&](uint32_t col, bool acc) {
    sm100::fence_proxy_async_smem();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    tmem = *reinterpret_cast<volatile uint32_t *>(smb + L::OMISC);
    if (tid == 0) {
      umma3_kmaj_mn<4>(tmem + col, sb + L::OAH, sb + L::OAL, L::A_BYTES, sb + L::OBH, sb + L::OBL, L::B_LBO,
                       IDESC, acc);
      sm100::mma_commit(bar_mma);
    }
  };
  float dot = 0.f;
  {  // D1 half 0: [dO; dU] and S0
    float xa[AI][8], xb[BI][8];
    ld_dodu(0, xa);
    ld_state(S0g, 0, xb);
    st_a_items(AH, AL, xa, tid);
    st_b_items<BI, DK, false>(BH, BL, L::B_LBO, xb, tid, dot);
  }
  issue(0, false);
  {  // D2 half 0: U and dS1 (loaded while D1 runs), <dS1, S0> over half 0
    float xa[UI][8], xb[BI][8];
    ld_u(0, xa);
    ld_state(S1g, 0, xb);
    cta_wait(bar_mma, 0, ctl, p.status);
    st_a_items(AH, AL, xa, tid);
    st_b_items<BI, DK, true>(BH, BL, L::B_LBO, xb, tid, dot);
  }
  issue(DK, false);
  if (NKH == 2) {
    {  // D2 half 1
      float xa[UI][8], xb[BI][8];
      ld_u(1, xa);
      ld_state(S1g, 1, xb);
      cta_wait(bar_mma, 1, ctl, p.status);
      st_a_items(AH, AL, xa, tid);
      st_b_items<BI, DK, false>(BH, BL, L::B_LBO, xb, tid, dot);
    }
    issue(DK, true);
    {  // D1 half 1, <S0, dS1> over half 1
      float xa[AI][8], xb[BI][8];
      ld_dodu(1, xa);
      ld_state(S0g, 1, xb);
      cta_wait(bar_mma, 0, ctl, p.status);
      st_a_items(AH, AL, xa, tid);
      st_b_items<BI, DK, true>(BH, BL, L::B_LBO, xb, tid, dot);
    }
    issue(0, true);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
  if (lane == 0) red[4 * C + w] = dot;
  // Epilogue: the finished accumulator first, then, after the last commit
  // (parity 1 in both orders), the other.  Warp w reads its rows and the
  // columns [half Dk / 2, + Dk / 2) in blocks of 32.
  const int qd = w & 3, half = w >> 2, row = 32 * qd + lane;
  const uint32_t tl = tmem + ((uint32_t)(32 * qd) << 16);
  const TI *q = static_cast<const TI *>(p.q), *k = static_cast<const TI *>(p.k);
  const size_t qoff = ((size_t)cp.start * p.Hqk + hk) * DK, qstride = (size_t)p.Hqk * DK;
  const float scale = p.scale;
  auto read_d1 = [&]() {
    float acc_g = 0.f;
    const float gam = row < len ? expf((float)sG[row < C ? row : 0]) : 0.f;
#pragma unroll
    for (int cc = 0; cc < DK / 64; ++cc) {
      const int col = half * (DK / 2) + 32 * cc;
      float v[32], qv[32];
      if (row < len) ld32(q + qoff + (size_t)row * qstride + col, qv);  // in flight beside the TMEM read
      sm100::tmem_ld32(tl + col, v);
      sm100::tmem_wait_ld();
      if (row < C) {  // dQ part and dgamma
        float *dst = p.dQp + (u * C + row) * DK + col;
#pragma unroll
        for (int x = 0; x < 32; x += 4) {
          *reinterpret_cast<float4 *>(dst + x) =
              make_float4(scale * gam * v[x], scale * gam * v[x + 1], scale * gam * v[x + 2], scale * gam * v[x + 3]);
          if (row < len)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc_g = fmaf(qv[x + e], v[x + e], acc_g);
        }
      } else {  // dW = -(dU S0)
        float *dst = p.dW + (u * C + row - C) * DK + col;
#pragma unroll
        for (int x = 0; x < 32; x += 4)
          *reinterpret_cast<float4 *>(dst + x) = make_float4(-v[x], -v[x + 1], -v[x + 2], -v[x + 3]);
      }
    }
    if (row < C) red[half * C + row] = scale * acc_g;
  };
  auto read_d2 = [&]() {
    if (qd >= 2) return;  // D2 rows 0-63: dK part and dkdec
    float acc_k = 0.f;
    const float kd = row < len ? expf((float)(sG[len - 1] - sG[row])) : 0.f;
#pragma unroll
    for (int cc = 0; cc < DK / 64; ++cc) {
      const int col = half * (DK / 2) + 32 * cc;
      float v[32], kv[32];
      if (row < len) ld32(k + qoff + (size_t)row * qstride + col, kv);  // in flight beside the TMEM read
      sm100::tmem_ld32(tl + DK + col, v);
      sm100::tmem_wait_ld();
      float *dst = p.dKp + (u * C + row) * DK + col;
#pragma unroll
      for (int x = 0; x < 32; x += 4) {
        *reinterpret_cast<float4 *>(dst + x) = make_float4(kd * v[x], kd * v[x + 1], kd * v[x + 2], kd * v[x + 3]);
        if (row < len)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc_k = fmaf(kv[x + e], v[x + e], acc_k);
      }
    }
    red[(2 + half) * C + row] = acc_k;
  };
  if (NKH == 2) {
    read_d2();
    cta_wait(bar_mma, 1, ctl, p.status);
    read_d1();
  } else {
    read_d1();
    cta_wait(bar_mma, 1, ctl, p.status);
    read_d2();
  }
  __syncthreads();
  float *sc = p.sc + u * 3 * C;
  if (tid < C) {
    sc[tid] = red[tid] + red[C + tid];
    sc[C + tid] = red[2 * C + tid] + red[3 * C + tid];
  }
  if (tid == 0) {
    float s = 0.f;
    for (int x = 0; x < NT / 32; ++x) s += red[4 * C + x];
    sc[2 * C] = s;
    // every MMA this thread issued has finished before the columns are freed
    sm100::mma_commit(bar_drain);
    sm100::mbar_wait_landed(bar_drain, 0, 50000000ull);
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (w == 0) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// ---- the 64 x 64 algebra of one (chunk, value head), and its outputs -----------
template <typename TI, int DK, int DV>
struct LocalSmem {
  static constexpr int DM = DK > DV ? DK : DV;
  static constexpr int LA = DM + 4;           // dO, then dW (fp32)
  static constexpr int LB = DV + 4;           // U, then dU (fp32)
  static constexpr int LC = in_ld<TI>(DK);    // K
  static constexpr int LD = in_ld<TI>(DM);    // V, then Q
  static constexpr size_t OA = 0, OB = OA + C * LA * 4, OC = OB + C * LB * 4,
                          OD = OC + up16(C * LC * sizeof(TI)), O1 = OD + up16(C * LD * sizeof(TI)),
                          O2 = O1 + C * LD64 * 4, O3 = O2 + C * LD64 * 4, O4 = O3 + C * LD64 * 4,
                          O5 = O4 + C * LD64 * 4, OG = O5 + C * LD64 * 4, OV = OG + 2 * C * 8,
                          NVEC = 11, BYTES = OV + NVEC * C * 4;
};

template <typename TI, int DK, int DV>
__global__ void __launch_bounds__(NT) grads_local_kernel(const Params p) {
  using L = LocalSmem<TI, DK, DV>;
  extern __shared__ __align__(16) unsigned char smb[];
  float *RA = reinterpret_cast<float *>(smb + L::OA), *RB = reinterpret_cast<float *>(smb + L::OB);
  TI *RC = reinterpret_cast<TI *>(smb + L::OC), *RD = reinterpret_cast<TI *>(smb + L::OD);
  float *S1 = reinterpret_cast<float *>(smb + L::O1), *S2 = reinterpret_cast<float *>(smb + L::O2),
        *S3 = reinterpret_cast<float *>(smb + L::O3), *S4 = reinterpret_cast<float *>(smb + L::O4),
        *S5 = reinterpret_cast<float *>(smb + L::O5);
  double *sGb = reinterpret_cast<double *>(smb + L::OG);  // G of this value head and the next
  float *vec = reinterpret_cast<float *>(smb + L::OV);
  // per-row vectors: beta, gamma, kdec, xk (2 halves), yv (2 halves), rP, cP, rM, cM
  float *sB = vec, *sGm = vec + C, *sKd = vec + 2 * C, *sXK = vec + 3 * C, *sYV = vec + 5 * C,
        *sRP = vec + 7 * C, *sCP = vec + 8 * C, *sRM = vec + 9 * C, *sCM = vec + 10 * C;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  ChunkPos cp;
  if (!chunk_pos(p, blockIdx.x, cp)) return;
  const int hk = blockIdx.y, Gq = p.Hv / p.Hqk;
  const int len = cp.len;
  const TI *q = static_cast<const TI *>(p.q), *k = static_cast<const TI *>(p.k),
           *v = static_cast<const TI *>(p.v);
  const size_t qoff = ((size_t)cp.start * p.Hqk + hk) * DK, qstride = (size_t)p.Hqk * DK;
  const float scale = p.scale;
  const int r0 = 16 * (w & 3), half = w >> 2, c64 = 32 * half;
  const int cbk = half * (DK / 2), cbv = half * (DV / 2);
  // dq and dk of the query/key head: the value heads of its group add their
  // parts in order, in registers
  float dQ[DK / 16][4], dK[DK / 16][4];
  zero_acc(dQ);
  zero_acc(dK);
  // dO, U, P, G and beta of value head gi + 1 are fetched while head gi
  // computes, each once its buffer is free (dO after the Y step, U after the
  // E.KK^T step, P after the row sums; G into the other of two buffers, beta
  // into a register)
  const float *dOg = p.dO + (size_t)cp.start * p.Hv * DV;
  const size_t dOs = (size_t)p.Hv * DV;
  float bnext = 0.f;
  for (int gi = 0; gi < Gq; ++gi) {
    const int h = hk * Gq + gi;
    const size_t u = (size_t)blockIdx.x * p.Hv + h;
    double *sG = sGb + (gi & 1) * C;
    if (gi == 0) {
      tile_async<C, DV>(RA, L::LA, dOg + (size_t)h * DV, dOs, len, tid);
      tile_async<C, DV>(RB, L::LB, p.U + u * C * DV, DV, C, tid);
      tile_async<C, C>(S1, LD64, p.P + u * C * C, C, C, tid);
      tile_async<1, C>(sG, C, p.G + u * C, 0, 1, tid);
    }
    cp_commit();
    if (gi == 0) tile_async<C, DK>(RC, L::LC, k + qoff, qstride, len, tid);  // K serves the group
    tile_async<C, DV>(RD, L::LD, v + ((size_t)cp.start * p.Hv + h) * DV, (size_t)p.Hv * DV, len, tid);
    tile_async<C, C>(S3, LD64, p.Tm + u * C * C, C, C, tid);
    cp_commit();
    if (tid < C) sB[tid] = gi > 0 ? bnext : tid < len ? p.beta[(size_t)(cp.start + tid) * p.Hv + h] : 0.f;
    float qp[DK / 16][4], kp[DK / 16][4];  // this head's state-gradient parts, in flight early
    frag_ld(qp, p.dQp + u * C * DK, DK, r0, cbk, lane);
    frag_ld(kp, p.dKp + u * C * DK, DK, r0, cbk, lane);
    cp_wait<1>();
    __syncthreads();
    if (tid < C) {
      sGm[tid] = tid < len ? expf((float)sG[tid]) : 0.f;
      sKd[tid] = tid < len ? expf((float)(sG[len - 1] - sG[tid])) : 0.f;
    }
    {  // step 1: dP = lower(dO' U^T); S2 = dP . E, S1 = dP . P
      float acc[4][4];
      zero_acc(acc);
      mma3_rows<DV>(acc, [&](int r, int c) { return RA[(r0 + r) * L::LA + c]; },
                        [&](int r, int c) { return RB[(c64 + c) * L::LB + r]; }, lane);
      for_frag(acc, r0, c64, lane, [&](int i, int j, float &x) {
        const float dp = i >= j ? scale * x : 0.f;
        S2[i * LD64 + j] = i >= j ? dp * expf((float)(sG[i] - sG[j])) : 0.f;
        S1[i * LD64 + j] = dp * S1[i * LD64 + j];
      });
    }
    __syncthreads();
    tile_async<C, DK>(RA, L::LA, p.dW + u * C * DK, DK, C, tid);
    tile_async<C, DV>(RB, L::LB, p.dU + u * C * DV, DV, C, tid);
    cp_commit();
    cp_wait<0>();
    __syncthreads();
    {  // step 2: dT = dW (diag(beta gamma) K)^T + dU (diag(beta) V)^T -> S4
      // (dW K^T and dU V^T with the raw inputs, then the column scales)
      constexpr bool EX = sizeof(TI) == 2;
      float a1[4][4], a2[4][4];
      zero_acc(a1);
      zero_acc(a2);
      mma3_rows<DK, 4, false, EX>(a1, [&](int r, int c) { return RA[(r0 + r) * L::LA + c]; },
                                       [&](int r, int c) { return to_f32(RC[(c64 + c) * L::LC + r]); }, lane);
      mma3_rows<DV, 4, false, EX>(a2, [&](int r, int c) { return RB[(r0 + r) * L::LB + c]; },
                                       [&](int r, int c) { return to_f32(RD[(c64 + c) * L::LD + r]); }, lane);
      const int tig = lane & 3;
#pragma unroll
      for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = r0 + gid + 8 * (e >> 1), j = c64 + 8 * t + 2 * tig + (e & 1);
          S4[i * LD64 + j] = sB[j] * (sGm[j] * a1[t][e] + a2[t][e]);
        }
    }
    {  // X = Tm^T dW; dK += diag(beta gamma) X
      float xa[DK / 16][4];
      zero_acc(xa);
      mma3_rows<C>(xa, [&](int r, int c) { return S3[c * LD64 + r0 + r]; },
                       [&](int r, int c) { return RA[r * L::LA + cbk + c]; }, lane);
      float slo, shi;
      quad_row_sums(xa, [&](int i, int c) { return to_f32(RC[i * L::LC + c]); }, r0, cbk, lane, slo, shi);
      if (tig == 0) { sXK[half * C + r0 + gid] = slo; sXK[half * C + r0 + gid + 8] = shi; }
#pragma unroll
      for (int t = 0; t < DK / 16; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = r0 + gid + 8 * (e >> 1);
          dK[t][e] = fmaf(sB[i] * sGm[i], xa[t][e], dK[t][e]);
        }
    }
    {  // Y = Tm^T dU: dv = diag(beta) Y
      float acc[DV / 16][4];
      zero_acc(acc);
      mma3_rows<C>(acc, [&](int r, int c) { return S3[c * LD64 + r0 + r]; },
                       [&](int r, int c) { return RB[r * L::LB + cbv + c]; }, lane);
      float slo, shi;
      quad_row_sums(acc, [&](int i, int c) { return to_f32(RD[i * L::LD + c]); }, r0, cbv, lane, slo, shi);
      if (tig == 0) { sYV[half * C + r0 + gid] = slo; sYV[half * C + r0 + gid + 8] = shi; }
      for_frag(acc, r0, cbv, lane, [&](int i, int c, float &x) { x *= sB[i]; });
      frag_st(acc, p.dv + ((size_t)cp.start * p.Hv + h) * DV, (size_t)p.Hv * DV, r0, cbv, lane, len);
    }
    __syncthreads();
    tile_async<C, DK>(RD, L::LD, q + qoff, qstride, len, tid);  // V is no longer needed
    tile_async<C, C>(RB, LD64, p.EKK + u * C * C, C, C, tid);   // dU is done with too
    if (gi + 1 < Gq) {
      tile_async<C, DV>(RA, L::LA, dOg + (size_t)(h + 1) * DV, dOs, len, tid);
      tile_async<1, C>(sGb + ((gi + 1) & 1) * C, C, p.G + (u + 1) * C, 0, 1, tid);
      if (tid < C) bnext = tid < len ? p.beta[(size_t)(cp.start + tid) * p.Hv + h + 1] : 0.f;
    }
    cp_commit();
    {  // Z = dT Tm^T -> S5
      float acc[4][4];
      zero_acc(acc);
      mma3_rows<C>(acc, [&](int r, int c) { return S4[(r0 + r) * LD64 + c]; },
                       [&](int r, int c) { return S3[(c64 + c) * LD64 + r]; }, lane);
      for_frag(acc, r0, c64, lane, [&](int i, int j, float &x) { S5[i * LD64 + j] = x; });
    }
    __syncthreads();
    {  // dA = strict_lower(-Tm^T Z) -> S4
      float acc[4][4];
      zero_acc(acc);
      mma3_rows<C>(acc, [&](int r, int c) { return S3[c * LD64 + r0 + r]; },
                       [&](int r, int c) { return S5[r * LD64 + c64 + c]; }, lane);
      for_frag(acc, r0, c64, lane, [&](int i, int j, float &x) { S4[i * LD64 + j] = i > j ? -x : 0.f; });
    }
    cp_wait<0>();
    __syncthreads();
    // S4 <- B = diag(beta) (dA . E); S5 <- dA . (E . K K^T), E . K K^T in RB
    for (int x = tid; x < C * C; x += NT) {
      const int i = x >> 6, j = x & 63;
      const float da = S4[i * LD64 + j];
      S4[i * LD64 + j] = i > j ? sB[i] * da * expf((float)(sG[i] - sG[j])) : 0.f;
      S5[i * LD64 + j] = da * RB[i * LD64 + j];
    }
    __syncthreads();
    if (gi + 1 < Gq) tile_async<C, DV>(RB, L::LB, p.U + (u + 1) * C * DV, DV, C, tid);
    cp_commit();
    if (tid < C) {  // row sums
      float a = 0.f, b = 0.f;
      for (int j = 0; j < C; ++j) { a += S1[tid * LD64 + j]; b += S5[tid * LD64 + j]; }
      sRP[tid] = a;
      sRM[tid] = b;
    } else if (tid < 2 * C) {  // column sums
      const int j = tid - C;
      float a = 0.f, b = 0.f;
      for (int i = 0; i < C; ++i) { a += S1[i * LD64 + j]; b += sB[i] * S5[i * LD64 + j]; }
      sCP[j] = a;
      sCM[j] = b;
    }
    {  // dq += diag(gamma) dO' S0 + (dP . E) K (this value head's parts)
#pragma unroll
      for (int t = 0; t < DK / 16; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) dQ[t][e] += qp[t][e];
      mma3_rows<C, DK / 16, false, sizeof(TI) == 2>(dQ, [&](int r, int c) { return S2[(r0 + r) * LD64 + c]; },
                       [&](int r, int c) { return to_f32(RC[r * L::LC + cbk + c]); }, lane);
    }
    {  // dk += diag(kdec) U dS1 + (dP . E)^T Q + (B + B^T) K (diag(beta gamma) X is in already)
#pragma unroll
      for (int t = 0; t < DK / 16; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) dK[t][e] += kp[t][e];
      mma3_rows<C, DK / 16, false, sizeof(TI) == 2>(dK, [&](int r, int c) { return S2[c * LD64 + r0 + r]; },
                       [&](int r, int c) { return to_f32(RD[r * L::LD + cbk + c]); }, lane);
      mma3_rows<C, DK / 16, false, sizeof(TI) == 2>(dK, [&](int r, int c) { return S4[(r0 + r) * LD64 + c] + S4[c * LD64 + r0 + r]; },
                       [&](int r, int c) { return to_f32(RC[r * L::LC + cbk + c]); }, lane);
    }
    __syncthreads();
    if (gi + 1 < Gq) tile_async<C, C>(S1, LD64, p.P + (u + 1) * C * C, C, C, tid);
    cp_commit();
    if (w == 0) {  // dG, then dg (suffix sums) and dbeta; two tokens per lane
      const float *sc = p.sc + u * 3 * C;
      const float dgC = sc[2 * C];
      float dG[2], db[2], kk2 = 0.f;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = 2 * lane + e;
        const float xk = sXK[i] + sXK[C + i], yv = sYV[i] + sYV[C + i];
        const float dgam = sc[i] + sB[i] * xk, dkd = sc[C + i];
        db[e] = sGm[i] * xk + yv + sRM[i];
        dG[e] = (sRP[i] - sCP[i]) + (sB[i] * sRM[i] - sCM[i]) + dgam * sGm[i] - dkd * sKd[i];
        kk2 += dkd * sKd[i];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) kk2 += __shfl_xor_sync(0xffffffffu, kk2, off);
      const float gC = expf((float)sG[len - 1]);
#pragma unroll
      for (int e = 0; e < 2; ++e)
        if (2 * lane + e == len - 1) dG[e] += kk2 + dgC * gC;
      // suffix sums over the chunk's tokens (rows >= len hold zeros)
      float s = dG[0] + dG[1];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float x = __shfl_down_sync(0xffffffffu, s, off);
        if (lane + off < 32) s += x;
      }
      const float sf[2] = {s, s - dG[0]};  // suffix from token 2 lane, from 2 lane + 1
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = 2 * lane + e;
        if (i < len) {
          p.dg[(size_t)(cp.start + i) * p.Hv + h] = sf[e];
          p.dbeta[(size_t)(cp.start + i) * p.Hv + h] = db[e];
        }
      }
    }
    __syncthreads();  // the next value head reuses every buffer but K
  }
  frag_st(dQ, p.dq + qoff, qstride, r0, cbk, lane, len);  // dq and dk of the query/key head
  frag_st(dK, p.dk + qoff, qstride, r0, cbk, lane, len);
}

}  // namespace cbwd

// Chunk-form backward workspace: header and plan, then the per-unit arrays.
struct CbwdLayout {
  size_t plan, Tm, P, EKK, W, dQp, dKp, dW, Ut, U, dU, S0, dS1, G, sc, total;
};

static CbwdLayout cbwd_layout(int64_t N, int64_t T, int Hqk, int Hv, int Dk, int Dv) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t units = (size_t)tp::chunk_bound(N, T) * Hv, f = sizeof(float), C = cbwd::C;
  CbwdLayout L;
  size_t o = kWorkspaceHeaderBytes;
  L.plan = o;  o += up(sizeof(int32_t) * (2 * (size_t)N + 1));
  L.Tm = o;    o += up(units * C * C * f);
  L.P = o;     o += up(units * C * C * f);
  L.EKK = o;   o += up(units * C * C * f);
  L.W = o;     o += up(units * C * Dk * f);
  L.dQp = o;   o += up(units * C * Dk * f);
  L.dKp = o;   o += up(units * C * Dk * f);
  L.dW = o;    o += up(units * C * Dk * f);
  L.Ut = o;    o += up(units * C * Dv * f);
  L.U = o;     o += up(units * C * Dv * f);
  L.dU = o;    o += up(units * C * Dv * f);
  L.S0 = o;    o += up(units * (size_t)Dv * Dk * f);
  L.dS1 = o;   o += up(units * (size_t)Dv * Dk * f);
  L.G = o;     o += up(units * C * sizeof(double));
  L.sc = o;    o += up(units * 3 * C * f);
  L.total = o;
  return L;
}

size_t backward_chunked_workspace_bytes(int64_t N, int64_t T, int Hqk, int Hv, int Dk, int Dv) {
  return cbwd_layout(N, T, Hqk, Hv, Dk, Dv).total;
}

namespace {

template <typename K>
cudaError_t launch_k(K kern, dim3 grid, size_t smem, const cbwd::Params &prm, cudaStream_t stream,
                     int threads = cbwd::NT) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (grid.x == 0 || grid.y == 0 || grid.z == 0) return cudaSuccess;
  kern<<<grid, threads, smem, stream>>>(prm);
  return cudaGetLastError();
}

template <typename TI, int DK, int DV>
cudaError_t run_chunked(const cbwd::Params &prm, int64_t chunks, cudaStream_t stream) {
  using namespace cbwd;
  constexpr size_t kMaxSmem = 232448;  // 227 KB, the most dynamic shared memory a CTA may use
  static_assert(PrepSmem<TI, DK, DV>::BYTES <= kMaxSmem && ChainSmem<TI, DK, DV>::BYTES <= kMaxSmem &&
                    StateGradSmem<DK, DV>::BYTES <= kMaxSmem && LocalSmem<TI, DK, DV>::BYTES <= kMaxSmem,
                "a backward kernel needs more shared memory than a CTA may use");
  const dim3 per_chunk((unsigned)chunks, (unsigned)prm.Hv);
  cudaError_t e;
  if ((e = launch_k(prep_kernel<TI, DK, DV>, per_chunk, PrepSmem<TI, DK, DV>::BYTES, prm, stream)) != cudaSuccess) return e;
  const dim3 chains((unsigned)(prm.N * prm.Hv * (DV / SL + 1)));
  if ((e = launch_k(chains_kernel<TI, DK, DV>, chains, ChainSmem<TI, DK, DV>::BYTES, prm, stream, NTR)) != cudaSuccess) return e;
  if ((e = launch_k(grads_state_kernel<TI, DK, DV>, per_chunk, StateGradSmem<DK, DV>::BYTES, prm, stream)) != cudaSuccess) return e;
  const dim3 per_group((unsigned)chunks, (unsigned)prm.Hqk);
  return launch_k(grads_local_kernel<TI, DK, DV>, per_group, LocalSmem<TI, DK, DV>::BYTES, prm, stream);
}

template <typename TI>
cudaError_t run_chunked_dims(const cbwd::Params &prm, int Dk, int Dv, int64_t chunks, cudaStream_t stream) {
  if (Dk == 128 && Dv == 128) return run_chunked<TI, 128, 128>(prm, chunks, stream);
  if (Dk == 128 && Dv == 64) return run_chunked<TI, 128, 64>(prm, chunks, stream);
  if (Dk == 64 && Dv == 128) return run_chunked<TI, 64, 128>(prm, chunks, stream);
  return run_chunked<TI, 64, 64>(prm, chunks, stream);
}

}  // namespace

cudaError_t launch_backward_chunked(const void *q, const void *k, const void *v, const float *g,
                                    const float *beta, const int32_t *cu, int N, long long T_, int Hqk,
                                    int Hv, int Dk, int Dv, int dtype, float scale, const float *s0,
                                    const float *dO, const float *dSfin, float *dq, float *dk,
                                    float *dv, float *dg, float *dbeta, float *ds0, void *workspace,
                                    cudaStream_t stream) {
  const int T = (int)T_;
  unsigned char *ws = static_cast<unsigned char *>(workspace);
  const CbwdLayout L = cbwd_layout(N, T, Hqk, Hv, Dk, Dv);
  int32_t *status = reinterpret_cast<int32_t *>(ws);
  auto *ph = reinterpret_cast<tp::PlanHeader *>(ws + tp::kPlanHeaderOffset);
  int32_t *ne_seq = reinterpret_cast<int32_t *>(ws + L.plan), *ne_cs = ne_seq + N;
  cudaError_t e = launch_plan(cu, N, T, Hv, dSfin, ds0, (size_t)Hv * Dv * Dk * sizeof(float), ph, ne_seq,
                              ne_cs, status, stream);
  if (e != cudaSuccess || T == 0) return e;
  auto F = [&](size_t off) { return reinterpret_cast<float *>(ws + off); };
  cbwd::Params prm;
  prm.q = q; prm.k = k; prm.v = v; prm.g = g; prm.beta = beta; prm.cu = cu;
  prm.N = N; prm.T = T; prm.Hqk = Hqk; prm.Hv = Hv; prm.scale = scale;
  prm.s0 = s0; prm.dO = dO; prm.dSf = dSfin;
  prm.dq = dq;
  prm.dk = dk;
  prm.dv = dv; prm.dg = dg; prm.dbeta = dbeta; prm.ds0 = ds0;
  prm.ph = ph; prm.ne_seq = ne_seq; prm.ne_cs = ne_cs;
  prm.Tm = F(L.Tm); prm.P = F(L.P); prm.EKK = F(L.EKK);
  prm.W = F(L.W); prm.dQp = F(L.dQp); prm.dKp = F(L.dKp); prm.dW = F(L.dW);
  prm.Ut = F(L.Ut); prm.U = F(L.U); prm.dU = F(L.dU);
  prm.S0 = F(L.S0); prm.dS1 = F(L.dS1); prm.sc = F(L.sc);
  prm.status = status;
  prm.G = reinterpret_cast<double *>(ws + L.G);
  const int64_t chunks = tp::chunk_bound(N, T);
  e = dtype == GDN_DTYPE_BF16 ? run_chunked_dims<__nv_bfloat16>(prm, Dk, Dv, chunks, stream)
                              : run_chunked_dims<float>(prm, Dk, Dv, chunks, stream);
  return e;
}

}  // namespace gdn
