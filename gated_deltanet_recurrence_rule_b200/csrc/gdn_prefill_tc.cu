// gdn_prefill_tc.cu -- chunked prefill of the gated delta rule on the
// Blackwell tensor cores (tcgen05 + TMEM + TMA), bf16 operands, fp32 state.
//
// The recurrence ("Inside Qwen3.8-27B: Hybrid DeltaNet Architecture, 256k
// Context, and 24GB Local Serving", section "Gated DeltaNet Mechanics"; the
// note there says prefill is rewritten into a block-parallel form for tensor
// cores while the state stays on chip):
//     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t.
// Chunked form for a chunk of C = 64 tokens with start state S0 (Dv x Dk),
// local log-decay prefix sums G_t and w_t = beta_t (v_t - alpha_t S_{t-1} k_t):
//     A_ts = beta_t e^{G_t - G_s} (k_t . k_s)   (s < t),   Tm = (I + A)^-1
//     W  = Tm diag(beta e^G) K,   U~ = Tm diag(beta) V,   U = U~ - W S0^T
//     O  = diag(e^G) Q S0^T + (e^{G_t - G_s} (q_t . k_s))_{s<=t} U
//     S  = e^{G_C} S0 + U^T diag(e^{G_C - G}) K
// Every product is computed transposed so that the 128-wide head dimension is
// the MMA's M (full-rate 128-lane tcgen05 tiles):
//     [Q;K] K^T        (M128 N64 K128)  -> QK^T and KK^T (exact bf16 inputs)
//     W^T  = K^T T'^T  (M128 N64 K64),  T'  = Tm diag(beta e^G)
//     U~^T = V^T T''^T (M128 N64 K64),  T'' = Tm diag(beta)
//     U^T  = U~^T - S0 W^T                   (accumulated with negated A)
//     Oi^T = S0 Q^T,   Oa^T = U^T P^T,   o_t = e^{G_t} Oi_t + Oa_t
//     dS   = (U diag(e^{G_C - G}))^T K,   S <- e^{G_C} S + dS  (fp32 master copy)
// Precision.  Rounding every operand to bf16 costs about 5e-2 RMS(o) in the
// largest output errors (the 1e-2 RMS bound needs ~11 significant bits at the
// largest outputs).  So the operands that carry computed values are split
// into two bf16 terms, x = hi + lo with hi = bf16(x), lo = bf16(x - hi):
// T' and T'' (2 MMAs each), S0 in the output product (2 MMAs), U and P in
// U^T P^T (hi*hi + lo*hi + hi*lo), and U diag(e^{G_C-G}) in dS (2 MMAs).  Q,
// K, V are exact bf16 inputs; decays are applied in fp32 (e^{G_t} on the
// output accumulator, e^{G_C-G_t} folded into U before the split).  S0 in
// U = U~ - W S0^T and W itself stay single bf16 (their rounding costs ~1e-3).
// The 64x64 unit lower-triangular inverse Tm is computed in fp32 on CUDA
// cores (16x16 diagonal blocks by forward substitution, then block rows).
//
// One CTA per (sequence, value head); 640 threads:
//   warp 0      TMA producer (Q/K ring of 2, V buffer of 1, L2 prefetch ahead)
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warp 2      per-chunk scalars (prefix sums of g, decays, masked beta)
//   warp 3      idle
//   warps 4-19  512 epilogue threads: TMEM -> registers -> SMEM operands,
//               the triangular solve, the fp32 state and the outputs.
// Chunks run one after another (this version does not overlap the next
// chunk's state-independent work with the current chunk's state chain).
// Every wait is bounded; a wait that runs out sets GDN_ERR_DEVICE_TIMEOUT in
// the workspace status word and every role leaves its loop.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "gdn_chunk_ops.cuh"
#include "gdn_common.cuh"
#include "gdn_sm100.cuh"
#include "gdn_twophase.cuh"

namespace gdn {
namespace tc {

using namespace sm100;
using namespace chunk;

constexpr int CH = 64;            // chunk length
constexpr int HD = 128;           // head dim (Dk = Dv)
constexpr int NTHREADS = 640;
constexpr int NEPI = 512;         // epilogue threads: 4 warpgroups, one quarter of the columns each
constexpr int EPI_BAR = 1;        // named barrier id of the epilogue threads
constexpr float LOG2E = 1.4426950408889634f;
// alpha below e^-30 is treated as e^-30: the chunk prefix sums stay finite
// (exp(-inf - -inf) is undefined) and e^-30 ~ 1e-13 is below fp32 resolution.
constexpr float G_FLOOR = -30.f;

// ---- shared memory map (bytes); swizzled tiles are 1024-byte aligned ----
constexpr int NQK = 3, NV = 2;          // ring depths (Q/K and V)
constexpr uint32_t QK_STAGE = 32768;   // [Q d0-63 | K d0-63 | Q d64-127 | K d64-127], 64 rows x 128 B each
constexpr uint32_t V_STAGE = 16384;    // [V d0-63 | V d64-127]
constexpr uint32_t OFF_QK = 0;
constexpr uint32_t OFF_V = OFF_QK + NQK * QK_STAGE;
// R1: a region reused by phases of a chunk that never overlap:
//   solve:   A fp32 [64][68] @0, Tm fp32 [64][68] @32K, Y fp32 [3][16][17] @50176
//   W, U~:   T' hi @0, T' lo @8K, T'' hi @16K, T'' lo @24K (Tm still read)
//   S0 W^T:  W^T bf16 MN-major (128 rows d x 64 t) @0
constexpr uint32_t OFF_R1 = OFF_V + NV * V_STAGE;
constexpr uint32_t OFF_A = OFF_R1;
constexpr uint32_t OFF_TM = OFF_R1 + 32768;
constexpr uint32_t OFF_Y = OFF_R1 + 50176;
constexpr uint32_t OFF_TPH = OFF_R1, OFF_TPL = OFF_R1 + 8192;
constexpr uint32_t OFF_TQH = OFF_R1 + 16384, OFF_TQL = OFF_R1 + 24576;
constexpr uint32_t OFF_WT = OFF_R1;
constexpr uint32_t R1_BYTES = 54272;
constexpr uint32_t OFF_PH = OFF_R1 + R1_BYTES;  // bf16 hi(P), K-major B: 64 rows (t) x 64 s
constexpr uint32_t OFF_PL = OFF_PH + 8192;      // bf16 lo(P)
constexpr uint32_t OFF_SCAL = OFF_PL + 8192;
constexpr uint32_t SCAL_STAGE = 7 * 64 * 4;  // G2 (log2 prefix), gamma, kdec, beta; gamma_C at [256]; 1/|q|, 1/|k| at [320], [384]
constexpr uint32_t OFF_BAR = OFF_SCAL + 2 * SCAL_STAGE;
constexpr uint32_t OFF_MISC = OFF_BAR + 192;  // [0] TMEM base, [4] control words (chunk::CTL_*), [16] drain mbarrier
constexpr uint32_t SMEM_BYTES = OFF_MISC + 24;
static_assert(OFF_R1 % 1024 == 0 && OFF_PH % 1024 == 0 && OFF_V % 1024 == 0, "alignment");
static_assert(OFF_Y + 3 * 16 * 17 * 4 <= OFF_R1 + R1_BYTES, "R1 layout");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// ---- TMEM columns (128 lanes x 512 columns of 32 bit) ----
// Accumulators (fp32) share columns across phases of a chunk that never overlap.
constexpr uint32_t R_QK = 0;    // 64: rows 0-63 = Q K^T, rows 64-127 = K K^T   (chunk start)
constexpr uint32_t R_W = 64;    // 64: W^T                                      (after the solve)
constexpr uint32_t R_S = 0;     // 128: dS                                      (chunk end)
constexpr uint32_t R_UO = 128;  // 64: U~^T, then U^T; afterwards U^T P^T
constexpr uint32_t R_OI = 192;  // 64: S0 Q^T
// MMA A operands in TMEM (bf16 pairs per column; lane = row of the operand).
constexpr uint32_t T_S0H = 256, T_S0L = 320;  // hi/lo(S0): 128 rows x 128 K (64 columns each)
constexpr uint32_t T_UH = 384, T_UL = 416;    // hi/lo(U^T): 128 rows x 64 K (32 columns each)
constexpr uint32_t T_UKH = 448, T_UKL = 480;  // hi/lo(U^T diag(kdec))
constexpr uint32_t TMEM_COLS = 512;

// ---- mbarriers ----
enum {
  B_FULL_QK = 0, B_EMPTY_QK = 3, B_FULL_V = 6, B_EMPTY_V = 8, B_SCAL_FULL = 10, B_SCAL_EMPTY = 12,
  B_QK = 14, B_T = 15, B_W = 16, B_WT = 17, B_U = 18, B_UT = 19, B_S = 20, B_DONE = 21, NBAR = 22
};
static_assert(NBAR * 8 <= 192, "barrier area");

constexpr uint32_t IDESC_QK = idesc_bf16(128, 64, 0, 0);      // [Q;K] K^T
constexpr uint32_t IDESC_WY = idesc_bf16(128, 64, 1, 0);      // K^T T'^T, V^T T''^T
constexpr uint32_t IDESC_SW = idesc_bf16(128, 64, 0, 1, 1);   // -S0 W^T
constexpr uint32_t IDESC_SQ = idesc_bf16(128, 64, 0, 0);      // S0 Q^T, U^T P^T
constexpr uint32_t IDESC_UK = idesc_bf16(128, 128, 0, 1);     // Ukdec^T K

struct Params {
  const float *g, *beta;
  const int32_t *cu;
  int N, T, Hqk, Hv;
  float scale;
  const void *s0;  // caller's initial states, fp32 or (state_bf16) bf16
  void *sfin;      // caller's final states, same type
  int state_bf16;
  int raw;         // GDN_INPUT_RAW: q, k normalised here, g and beta through -softplus, sigmoid
  const void *q, *k;  // raw inputs: rows read for their norms
  void *o;
  int32_t *status;
};

__device__ __forceinline__ uint32_t bar_addr(uint32_t sb, int i) { return sb + OFF_BAR + 8u * i; }

__device__ __forceinline__ bool epi_wait(uint32_t bar, uint32_t parity, int etid,
                                         volatile int *ctl, int32_t *status) {
  return group_wait<NEPI, EPI_BAR>(bar, parity, etid, ctl, status);
}

template <typename TO>
__global__ void __launch_bounds__(NTHREADS, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x / p.Hv, h = blockIdx.x - n * p.Hv;
  const int j = h / (p.Hv / p.Hqk);
  const size_t sbase = ((size_t)n * p.Hv + h) * HD * HD;

  const int c0 = p.cu[n], c1 = p.cu[n + 1];
  if (c0 < 0 || c1 < c0 || c1 > p.T || (n == 0 && c0 != 0) || (n == p.N - 1 && c1 != p.T)) {
    if (tid == 0) report_status(p.status, GDN_ERR_BAD_SEQLENS);
    return;
  }
  const int L = c1 - c0;
  const int nch = (L + CH - 1) / CH;
  if (nch == 0) {  // empty sequence: final state = initial state (a byte copy)
    if (p.sfin) {
      const int eb = p.state_bf16 ? 2 : 4;
      uint4 *dst = reinterpret_cast<uint4 *>(static_cast<unsigned char *>(p.sfin) + sbase * eb);
      const uint4 *src = p.s0 ? reinterpret_cast<const uint4 *>(
                                    static_cast<const unsigned char *>(p.s0) + sbase * eb)
                              : nullptr;
      for (int x = tid; x < HD * HD * eb / 16; x += NTHREADS)
        dst[x] = src ? src[x] : make_uint4(0u, 0u, 0u, 0u);
    }
    return;
  }

  const uint32_t sb = smem_addr(smem);
  if (sb & 1023u) {  // swizzled operand tiles need 1024-byte alignment
    if (tid == 0) report_status(p.status, GDN_ERR_UNSUPPORTED);
    return;
  }
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
  if (tid == 0) {
    for (int i = 0; i < NBAR; ++i) mbar_init(bar_addr(sb, i), 1);
    abort_flag[CTL_ABORT] = 0;
    abort_flag[CTL_LIMIT] = 0;  // 2 s until warp 3 has read the header
    abort_flag[CTL_GROUP] = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(sb + OFF_MISC, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + OFF_MISC);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      constexpr int PF = 4;  // L2 prefetch distance in chunks
      for (int c = 0; c < PF && c < nch; ++c) {
        const int t = c0 + c * CH;
        tma_prefetch_3d(&tm_q, 0, j, t); tma_prefetch_3d(&tm_q, 64, j, t);
        tma_prefetch_3d(&tm_k, 0, j, t); tma_prefetch_3d(&tm_k, 64, j, t);
        tma_prefetch_3d(&tm_v, 0, h, t); tma_prefetch_3d(&tm_v, 64, h, t);
      }
      int issued_qk = 0, issued_v = 0;  // chunks whose loads were issued
      for (int c = 0; c < nch; ++c) {
        const int s = c % NQK, sv = c % NV;
        const int t0 = c0 + c * CH;
        if (c + PF < nch) {
          const int t = t0 + PF * CH;
          tma_prefetch_3d(&tm_q, 0, j, t); tma_prefetch_3d(&tm_q, 64, j, t);
          tma_prefetch_3d(&tm_k, 0, j, t); tma_prefetch_3d(&tm_k, 64, j, t);
          tma_prefetch_3d(&tm_v, 0, h, t); tma_prefetch_3d(&tm_v, 64, h, t);
        }
        if (!mbar_wait(bar_addr(sb, B_EMPTY_QK + s), ((c / NQK) & 1) ^ 1, abort_flag)) break;
        const uint32_t st = sb + OFF_QK + s * QK_STAGE;
        const uint32_t fb = bar_addr(sb, B_FULL_QK + s);
        mbar_arrive_expect_tx(fb, QK_STAGE);
        tma_load_3d(st + 0, &tm_q, fb, 0, j, t0);
        tma_load_3d(st + 16384, &tm_q, fb, 64, j, t0);
        tma_load_3d(st + 8192, &tm_k, fb, 0, j, t0);
        tma_load_3d(st + 24576, &tm_k, fb, 64, j, t0);
        issued_qk = c + 1;
        if (!mbar_wait(bar_addr(sb, B_EMPTY_V + sv), ((c / NV) & 1) ^ 1, abort_flag)) break;
        const uint32_t vs = sb + OFF_V + sv * V_STAGE;
        const uint32_t fv = bar_addr(sb, B_FULL_V + sv);
        mbar_arrive_expect_tx(fv, V_STAGE);
        tma_load_3d(vs + 0, &tm_v, fv, 0, h, t0);
        tma_load_3d(vs + 8192, &tm_v, fv, 64, h, t0);
        issued_v = c + 1;
      }
      if (issued_qk < nch || issued_v < nch) {
        *abort_flag = 1;
        report_status(p.status, GDN_ERR_DEVICE_TIMEOUT);
      }
      // Let every load this thread issued land before the CTA can exit (each
      // buffer's latest fill; earlier fills were consumed before it was issued).
      for (int c = max(issued_qk - NQK, 0); c < issued_qk; ++c)
        mbar_wait_landed(bar_addr(sb, B_FULL_QK + c % NQK), (c / NQK) & 1, 50000000ull);
      for (int c = max(issued_v - NV, 0); c < issued_v; ++c)
        mbar_wait_landed(bar_addr(sb, B_FULL_V + c % NV), (c / NV) & 1, 50000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Base descriptors, built once; per-MMA offsets are compile-time byte
      // counts added to the start-address field (bytes / 16).
      const uint64_t dQK0 = sdesc_sw128(sb + OFF_QK, 16, 1024);            // Q/K stage, K-major
      const uint64_t dKmn0 = sdesc_sw128(sb + OFF_QK + 8192, 16384, 1024); // K as MN-major operand
      const uint64_t dVmn0 = sdesc_sw128(sb + OFF_V, 8192, 1024);           // V as MN-major operand
      const uint64_t dR1 = sdesc_sw128(sb + OFF_R1, 16, 1024);              // T splits (K-major)
      const uint64_t dWT = sdesc_sw128(sb + OFF_WT, 8192, 1024);            // W^T, MN-major
      const uint64_t dP = sdesc_sw128(sb + OFF_PH, 16, 1024);               // P hi / lo, K-major
      bool ok = true;
      for (int c = 0; c < nch && ok; ++c) {
        const int s = c % NQK, sv = c % NV;
        const uint32_t ph = c & 1;
        const uint64_t dQK = dQK0 + s * (QK_STAGE >> 4), dKmn = dKmn0 + s * (QK_STAGE >> 4);
        const uint64_t dVmn = dVmn0 + sv * (V_STAGE >> 4);
        // [Q;K] K^T
        ok = mbar_wait(bar_addr(sb, B_FULL_QK + s), (c / NQK) & 1, abort_flag);
        if (ok && c > 0) ok = mbar_wait(bar_addr(sb, B_DONE), (c - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t k16 = ((ks >> 2) * 16384 + (ks & 3) * 32) >> 4;
          mma_bf16(tmem + R_QK, dQK + k16, dQK + (8192 >> 4) + k16, IDESC_QK, ks > 0);
        }
        mma_commit(bar_addr(sb, B_QK));
        // W^T = K^T (T'h + T'l)^T ;  U~^T = V^T (T''h + T''l)^T
        ok = mbar_wait(bar_addr(sb, B_T), ph, abort_flag) &&
             mbar_wait(bar_addr(sb, B_FULL_V + sv), (c / NV) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t bo = (((ks & 1) ? OFF_TPL : OFF_TPH) - OFF_R1 + (ks >> 1) * 32) >> 4;
          mma_bf16(tmem + R_W, dKmn + (((ks >> 1) * 2048) >> 4), dR1 + bo, IDESC_WY, ks > 0);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t bo = (((ks & 1) ? OFF_TQL : OFF_TQH) - OFF_R1 + (ks >> 1) * 32) >> 4;
          mma_bf16(tmem + R_UO, dVmn + (((ks >> 1) * 2048) >> 4), dR1 + bo, IDESC_WY, ks > 0);
        }
        mma_commit(bar_addr(sb, B_W));
        mma_commit(bar_addr(sb, B_EMPTY_V + sv));
        // U^T = U~^T - S0h W^T ;  Oi^T = (S0h + S0l) Q^T   (S0 from TMEM)
        ok = mbar_wait(bar_addr(sb, B_WT), ph, abort_flag);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ts(tmem + R_UO, tmem + T_S0H + 8 * ks, dWT + ((ks * 2048) >> 4), IDESC_SW, 1);
#pragma unroll
        for (int ks = 0; ks < 16; ++ks) {
          const int k = ks >> 1;
          const uint32_t k16 = ((k >> 2) * 16384 + (k & 3) * 32) >> 4;
          mma_bf16_ts(tmem + R_OI, tmem + ((ks & 1) ? T_S0L : T_S0H) + 8 * k, dQK + k16, IDESC_SQ,
                      ks > 0);
        }
        mma_commit(bar_addr(sb, B_U));
        // dS = (Ukh + Ukl)^T K ;  Oa^T = Uh Ph^T + Ul Ph^T + Uh Pl^T   (U from TMEM)
        ok = mbar_wait(bar_addr(sb, B_UT), ph, abort_flag);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const int kk = ks >> 1;
          mma_bf16_ts(tmem + R_S, tmem + ((ks & 1) ? T_UKL : T_UKH) + 8 * kk,
                      dKmn + ((kk * 2048) >> 4), IDESC_UK, ks > 0);
        }
#pragma unroll
        for (int ks = 0; ks < 12; ++ks) {
          const int part = ks % 3, kk = ks / 3;  // (Uh,Ph), (Ul,Ph), (Uh,Pl)
          const uint32_t bo = ((part == 2 ? OFF_PL - OFF_PH : 0) + kk * 32) >> 4;
          mma_bf16_ts(tmem + R_UO, tmem + (part == 1 ? T_UL : T_UH) + 8 * kk, dP + bo, IDESC_SQ,
                      ks > 0);
        }
        mma_commit(bar_addr(sb, B_S));
        mma_commit(bar_addr(sb, B_EMPTY_QK + s));
      }
      if (!ok) {
        *abort_flag = 1;
        report_status(p.status, GDN_ERR_DEVICE_TIMEOUT);
      }
      // Drain: every MMA this thread issued finishes before TMEM is freed.
      const uint32_t drain = sb + OFF_MISC + 16;
      mbar_init(drain, 1);
      fence_barrier_init();
      mma_commit(drain);
      mbar_wait_landed(drain, 0, 50000000ull);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ chunk scalars
    for (int c = 0; c < nch; ++c) {
      const int s = c & 1;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(bar_addr(sb, B_SCAL_EMPTY + s), ((c >> 1) & 1) ^ 1, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) { *abort_flag = 1; report_status(p.status, GDN_ERR_DEVICE_TIMEOUT); }
        break;
      }
      const int t0 = c0 + c * CH;
      const int Lc = min(CH, c1 - t0);
      float ga = 0.f, gb = 0.f, ba = 0.f, bb = 0.f;
      auto log_alpha = [&](float x) { return fmaxf(p.raw ? log_alpha_raw(x) : x, G_FLOOR); };
      auto write_strength = [&](float x) { return p.raw ? beta_raw(x) : x; };
      if (lane < Lc) {
        ga = log_alpha(p.g[(size_t)(t0 + lane) * p.Hv + h]);
        ba = write_strength(p.beta[(size_t)(t0 + lane) * p.Hv + h]);
      }
      if (lane + 32 < Lc) {
        gb = log_alpha(p.g[(size_t)(t0 + lane + 32) * p.Hv + h]);
        bb = write_strength(p.beta[(size_t)(t0 + lane + 32) * p.Hv + h]);
      }
      // Raw inputs: 1/|q_t|, 1/|k_t| of rows t = lane, lane + 32 (read from global
      // memory: the shared tiles are recycled once their MMAs are done), folded
      // into the scalars below and in the epilogue, not into the bf16 tiles.
      float rq[2] = {1.f, 1.f}, rk[2] = {1.f, 1.f};
      if (p.raw) {
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int t = lane + 32 * w;
          float sq = 0.f, sk = 0.f;
          if (t < Lc) {
            const size_t off = ((size_t)(t0 + t) * p.Hqk + j) * HD;
            const uint4 *qr = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.q) + off);
            const uint4 *kr = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.k) + off);
#pragma unroll 4
            for (int c16 = 0; c16 < HD / 8; ++c16) {
              const uint4 xq = qr[c16], xk = kr[c16];
              const uint32_t wq[4] = {xq.x, xq.y, xq.z, xq.w}, wk[4] = {xk.x, xk.y, xk.z, xk.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float q0 = __uint_as_float(wq[i] << 16), q1 = __uint_as_float(wq[i] & 0xffff0000u);
                const float k0 = __uint_as_float(wk[i] << 16), k1 = __uint_as_float(wk[i] & 0xffff0000u);
                sq = fmaf(q0, q0, fmaf(q1, q1, sq));
                sk = fmaf(k0, k0, fmaf(k1, k1, sk));
              }
            }
          }
          rq[w] = inv_norm(sq);
          rk[w] = inv_norm(sk);
        }
      }
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float xa = __shfl_up_sync(0xffffffffu, ga, off);
        const float xb = __shfl_up_sync(0xffffffffu, gb, off);
        if (lane >= off) { ga += xa; gb += xb; }
      }
      gb += __shfl_sync(0xffffffffu, ga, 31);
      const float Ga = ga * LOG2E, Gb = gb * LOG2E;  // log2 of the decay prefix
      const int last = Lc - 1;
      const float GL = last < 32 ? __shfl_sync(0xffffffffu, Ga, last & 31)
                                 : __shfl_sync(0xffffffffu, Gb, last & 31);
      float *sc = reinterpret_cast<float *>(smem + OFF_SCAL + s * SCAL_STAGE);
      sc[lane] = Ga;                 sc[lane + 32] = Gb;
      sc[64 + lane] = exp2f(Ga);     sc[64 + lane + 32] = exp2f(Gb);
      sc[128 + lane] = lane < Lc ? exp2f(GL - Ga) * rk[0] : 0.f;
      sc[128 + lane + 32] = lane + 32 < Lc ? exp2f(GL - Gb) * rk[1] : 0.f;
      sc[192 + lane] = ba;           sc[192 + lane + 32] = bb;
      if (lane == 0) sc[256] = exp2f(GL);
      sc[320 + lane] = rq[0];        sc[320 + lane + 32] = rq[1];
      sc[384 + lane] = rk[0];        sc[384 + lane + 32] = rk[1];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_addr(sb, B_SCAL_FULL + s));
    }
  } else if (warp == 3) {
    // the caller's wait limit (a global load kept off the other roles' start)
    if (lane == 0) abort_flag[CTL_LIMIT] = (int)header_wait_limit_us(p.status);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int etid = tid - 128;
    const int ewq = etid >> 7;         // column quarter
    const int row = etid & 127;        // TMEM lane = row of the 128-row tiles
    const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    float *A = reinterpret_cast<float *>(smem + OFF_A);
    float *Tm = reinterpret_cast<float *>(smem + OFF_TM);
    float *Y = reinterpret_cast<float *>(smem + OFF_Y);

    // fp32 master state: row `row`, columns [32 ewq, 32 ewq + 32); S0 = hi + lo in TMEM
    float S[32];
    {
      const size_t e0 = sbase + (size_t)row * HD + 32 * ewq;
#pragma unroll
      for (int x = 0; x < 32; x += 4) {
        if (p.s0) load_state4(p.s0, e0 + x, p.state_bf16, S + x);
        else S[x] = S[x + 1] = S[x + 2] = S[x + 3] = 0.f;
      }
      uint32_t hw[16], lw[16];
      split_words<16>(S, hw, lw);
      tmem_st16(tl + T_S0H + 16 * ewq, hw);
      tmem_st16(tl + T_S0L + 16 * ewq, lw);
      tmem_wait_st();
    }

    for (int c = 0; c < nch; ++c) {
      const int s = c & 1;
      const uint32_t ph = c & 1;
      const int t0 = c0 + c * CH;
      const int Lc = min(CH, c1 - t0);
      const float *sc = reinterpret_cast<const float *>(smem + OFF_SCAL + s * SCAL_STAGE);
      const float *G2 = sc, *gam = sc + 64, *kdec = sc + 128, *bet = sc + 192, *rqn = sc + 320,
                  *rkn = sc + 384;

      // ---- Q K^T and K K^T -> P (hi/lo) and A (fp32)
      if (etid == 0) {
        if (!mbar_wait(bar_addr(sb, B_SCAL_FULL + s), (c >> 1) & 1, abort_flag)) {
          abort_flag[CTL_ABORT] = 1;
          abort_flag[CTL_GROUP] = 1;  // the group's waiter: the next group wait gives up
          report_status(p.status, GDN_ERR_DEVICE_TIMEOUT);
        }
      }
      if (!epi_wait(bar_addr(sb, B_QK), ph, etid, abort_flag, p.status)) break;
      {
        float v[16];
        tmem_ld16(tl + R_QK + 16 * ewq, v);
        tmem_wait_ld();
        if (row < 64) {
          const int t = row;
          const float Gt = G2[t], rq = rqn[t];
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            float pv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int si = 16 * ewq + 8 * q + e;
              pv[e] = (si <= t && t < Lc) ? exp2f(Gt - G2[si]) * v[8 * q + e] * (rq * rkn[si]) : 0.f;
            }
            const uint32_t off = sw128_off(t, 2 * ewq + q);
            st_split8(smem + OFF_PH + off, smem + OFF_PL + off, pv);
          }
        } else {
          const int t = row - 64;
          const float Gt = G2[t], bt = bet[t], rk = rkn[t];
          float *arow = A + t * AST + 16 * ewq;
#pragma unroll
          for (int x = 0; x < 16; x += 4) {
            float a[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int si = 16 * ewq + x + e;
              a[e] = (si < t && t < Lc) ? bt * exp2f(Gt - G2[si]) * v[x + e] * (rk * rkn[si]) : 0.f;
            }
            *reinterpret_cast<float4 *>(arow + x) = make_float4(a[0], a[1], a[2], a[3]);
          }
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(EPI_BAR, NEPI);

      // ---- Tm = (I + A)^-1, then T' = Tm diag(beta gamma), T'' = Tm diag(beta), split
      ut_solve<NEPI, EPI_BAR>(A, Tm, Y, etid);
      {
        const int t = etid >> 3, sbeg = 8 * (etid & 7);
        float tm[8], bt[8], gm[8], tp[8], tq[8];
#pragma unroll
        for (int e = 0; e < 8; e += 4) {
          const float4 a4 = *reinterpret_cast<const float4 *>(Tm + t * AST + sbeg + e);
          const float4 b4 = *reinterpret_cast<const float4 *>(bet + sbeg + e);
          const float4 g4 = *reinterpret_cast<const float4 *>(gam + sbeg + e);
          const float4 r4 = *reinterpret_cast<const float4 *>(rkn + sbeg + e);
          tm[e] = a4.x; tm[e + 1] = a4.y; tm[e + 2] = a4.z; tm[e + 3] = a4.w;
          bt[e] = b4.x; bt[e + 1] = b4.y; bt[e + 2] = b4.z; bt[e + 3] = b4.w;
          gm[e] = g4.x * r4.x; gm[e + 1] = g4.y * r4.y; gm[e + 2] = g4.z * r4.z; gm[e + 3] = g4.w * r4.w;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float m = (sbeg + e <= t) ? tm[e] : 0.f;
          tq[e] = m * bt[e];
          tp[e] = tq[e] * gm[e];
        }
        const uint32_t off = sw128_off(t, sbeg >> 3);
        st_split8(smem + OFF_TPH + off, smem + OFF_TPL + off, tp);
        st_split8(smem + OFF_TQH + off, smem + OFF_TQL + off, tq);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(EPI_BAR, NEPI);
      if (etid == 0) mbar_arrive(bar_addr(sb, B_T));

      // ---- W^T -> bf16 (MN-major B)
      if (!epi_wait(bar_addr(sb, B_W), ph, etid, abort_flag, p.status)) break;
      {
        float v[16];
        tmem_ld16(tl + R_W + 16 * ewq, v);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 2; ++q) st_bf16x8(smem + OFF_WT + sw128_off(row, 2 * ewq + q), v + 8 * q);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(EPI_BAR, NEPI);
      if (etid == 0) mbar_arrive(bar_addr(sb, B_WT));

      // ---- U^T -> hi/lo (for P) and U^T diag(kdec) -> hi/lo (for the state), into TMEM
      if (!epi_wait(bar_addr(sb, B_U), ph, etid, abort_flag, p.status)) break;
      {
        float v[16];
        tmem_ld16(tl + R_UO + 16 * ewq, v);
        tmem_wait_ld();
        uint32_t hw[8], lw[8];
        split_words<8>(v, hw, lw);
        tmem_st8(tl + T_UH + 8 * ewq, hw);
        tmem_st8(tl + T_UL + 8 * ewq, lw);
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] *= kdec[16 * ewq + e];
        split_words<8>(v, hw, lw);
        tmem_st8(tl + T_UKH + 8 * ewq, hw);
        tmem_st8(tl + T_UKL + 8 * ewq, lw);
        tmem_wait_st();
      }
      tc_fence_before();
      named_bar_sync(EPI_BAR, NEPI);
      if (etid == 0) mbar_arrive(bar_addr(sb, B_UT));

      // ---- state: S = gamma_C S + dS (fp32), S0 <- hi/lo(S); outputs
      if (!epi_wait(bar_addr(sb, B_S), ph, etid, abort_flag, p.status)) break;
      {
        const float gC = sc[256];
        {
          float v[32];
          tmem_ld32(tl + R_S + 32 * ewq, v);
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x) S[x] = fmaf(gC, S[x], v[x]);
        }
        {
          uint32_t hw[16], lw[16];
          split_words<16>(S, hw, lw);
          tmem_st16(tl + T_S0H + 16 * ewq, hw);
          tmem_st16(tl + T_S0L + 16 * ewq, lw);
        }
        float vi[16], va[16];
        tmem_ld16(tl + R_OI + 16 * ewq, vi);
        tmem_ld16(tl + R_UO + 16 * ewq, va);
        tmem_wait_ld();
        TO *op = static_cast<TO *>(p.o) + ((size_t)t0 * p.Hv + h) * HD + row;
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const int t = 16 * ewq + x;
          if (t < Lc) op[(size_t)t * p.Hv * HD] = from_f32<TO>(p.scale * fmaf(gam[t] * rqn[t], vi[x], va[x]));
        }
        tmem_wait_st();
      }
      tc_fence_before();
      named_bar_sync(EPI_BAR, NEPI);
      if (etid == 0) {
        mbar_arrive(bar_addr(sb, B_DONE));
        mbar_arrive(bar_addr(sb, B_SCAL_EMPTY + s));
      }
    }
    if (*abort_flag == 0 && p.sfin) {
      const size_t e0 = sbase + (size_t)row * HD + 32 * ewq;
#pragma unroll
      for (int x = 0; x < 32; x += 4) store_state4(p.sfin, e0 + x, p.state_bf16, S + x);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <typename TO>
static cudaError_t launch_t(const void *q, const void *k, const void *v, const Params &prm,
                            cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  if (!make_qkv_map(&mq, q, prm.Hqk, prm.T) || !make_qkv_map(&mk, k, prm.Hqk, prm.T) ||
      !make_qkv_map(&mv, v, prm.Hv, prm.T))
    return cudaErrorInvalidValue;
  auto kern = prefill_tc_kernel<TO>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)prm.N * (unsigned)prm.Hv, NTHREADS, SMEM_BYTES, stream>>>(mq, mk, mv, prm);
  return cudaGetLastError();
}

}  // namespace tc

bool prefill_tc_supported(int Hqk, int Hv, int Dk, int Dv, int dtype) {
  return dtype == GDN_DTYPE_BF16 && Dk == 128 && Dv == 128 && Hqk > 0 && Hv % Hqk == 0;
}

cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const int32_t *cu, int N, long long T_, int Hqk,
                              int Hv, int o_dtype, int state_dtype, int input_form, float scale,
                              const void *s0, void *sfin, void *o, void *workspace,
                              cudaStream_t stream) {
  tc::Params prm;
  prm.raw = input_form == GDN_INPUT_RAW;
  prm.q = q; prm.k = k;
  prm.g = g; prm.beta = beta; prm.cu = cu; prm.N = N; prm.T = (int)T_; prm.Hqk = Hqk; prm.Hv = Hv;
  prm.scale = scale; prm.s0 = s0; prm.sfin = sfin; prm.state_bf16 = state_dtype == GDN_DTYPE_BF16;
  prm.o = o;
  prm.status = static_cast<int32_t *>(workspace);
  if (o_dtype == GDN_DTYPE_BF16) return tc::launch_t<__nv_bfloat16>(q, k, v, prm, stream);
  return tc::launch_t<float>(q, k, v, prm, stream);
}

}  // namespace gdn
