// gdn_wy_prep.cu -- phase 1 of the two-phase tensor-core prefill: the
// state-free products of every (chunk, value head) at once.
//
// For a chunk of C = 64 tokens (aligned to its sequence start) and value head
// h reading query/key head j = h / (Hv / Hqk), with local log-decay prefix sums
// G_t = sum_{s <= t} g_s ("Inside Qwen3.8-27B: Hybrid DeltaNet Architecture,
// 256k Context, and 24GB Local Serving", section "Gated DeltaNet Mechanics":
// the decay alpha_t = e^{g_t} scales the whole state, beta_t the write):
//     [Q;K] K^T                 one M128 N64 K128 MMA: rows 0-63 Q K^T, 64-127 K K^T
//     P_ts = e^{G_t-G_s} q_t.k_s (s <= t)          -> record, bf16 hi + lo
//     A_ts = beta_t e^{G_t-G_s} k_t.k_s (s < t)    -> shared memory, fp32
//     Tm = (I + A)^-1                              fp32 on CUDA cores
//     T' = Tm diag(beta e^G),  T'' = Tm diag(beta) -> bf16 hi + lo operand tiles
//     W^T  = K^T T'^T   (M128 N64 K64, 2 MMAs per K step: hi and lo of T')
//     U~^T = V^T T''^T  (same shape)
//     W^T -> record as bf16, U~ -> record as fp32, with e^{G_t},
//     e^{G_C - G_t} and e^{G_C}.
// With raw inputs (GDN_INPUT_RAW) g and beta pass through -softplus and
// sigmoid here, and q, k are normalised by folding 1/|q_t|, 1/|k_t| into the
// per-token scalars (the operand tiles keep the raw bf16 values).
// Padded rows (t >= chunk length) get beta = 0, so their W and U~ rows are 0.
//
// One CTA per (chunk of the round, value head), two CTAs per SM; 384 threads:
//   warp 0      TMA loads of the Q/K and V tiles
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warp 2      chunk scalars (prefix sums, decays, masked beta)
//   warps 4-11  256 epilogue threads: TMEM -> P / A, the triangular solve,
//               the T' / T'' splits and the W^T / U~ stores.
// Every wait is bounded; a wait that runs out sets GDN_ERR_DEVICE_TIMEOUT.
#include <cuda.h>

#include "gdn_chunk_ops.cuh"
#include "gdn_common.cuh"
#include "gdn_sm100.cuh"
#include "gdn_twophase.cuh"

namespace gdn {
namespace wy {

using namespace sm100;
using namespace chunk;
using tp::CH;
using tp::HD;

constexpr int NTHREADS = 384;
constexpr int NEPI = 256;
constexpr int EPI_BAR = 1;
constexpr float LOG2E = 1.4426950408889634f;
// alpha below e^-30 is treated as e^-30 so that the chunk prefix sums stay
// finite; e^-30 ~ 1e-13 is below fp32 resolution of the state.
constexpr float G_FLOOR = -30.f;

// ---- shared memory map (bytes) ----
constexpr uint32_t OFF_QK = 0;       // [Q d0-63 | K d0-63 | Q d64-127 | K d64-127], 64 rows x 128 B each
constexpr uint32_t OFF_V = 32768;    // [V d0-63 | V d64-127]
constexpr uint32_t OFF_R1 = 49152;
constexpr uint32_t OFF_A = OFF_R1;             // fp32 [64][AST]
constexpr uint32_t OFF_TM = OFF_R1 + 17408;    // fp32 [64][AST]
constexpr uint32_t OFF_Y = OFF_R1 + 34816;     // fp32 [3][16][17]
constexpr uint32_t OFF_TPH = OFF_R1;           // hi/lo(T') over A, after the solve
constexpr uint32_t OFF_TPL = OFF_R1 + 8192;
constexpr uint32_t OFF_TQH = OFF_QK;           // hi/lo(T'') over the Q halves, after [Q;K]K^T
constexpr uint32_t OFF_TQL = OFF_QK + 16384;
constexpr uint32_t OFF_SCAL = OFF_R1 + 38912;  // G2 (log2 prefix), gamma, kdec, beta, 1/|q|, 1/|k| [64 each]
constexpr uint32_t OFF_BAR = OFF_SCAL + 1792;
constexpr uint32_t OFF_MISC = OFF_BAR + 64;    // [0] TMEM base, [4] control words (chunk::CTL_*), [16] drain mbarrier
constexpr uint32_t SMEM_BYTES = OFF_MISC + 24;
static_assert(OFF_Y + 3 * 16 * 17 * 4 <= OFF_SCAL, "R1 layout");
static_assert(OFF_R1 % 1024 == 0 && OFF_TPL % 1024 == 0 && OFF_V % 1024 == 0, "alignment");
static_assert(2 * SMEM_BYTES <= 232448 - 2048, "two CTAs per SM");

enum { B_QKF = 0, B_VF, B_SCAL, B_QK, B_T, B_W, NBAR };
static_assert(NBAR * 8 <= 64, "barrier area");

// TMEM columns (fp32 accumulators, 128 lanes)
constexpr uint32_t R_QK = 0, R_W = 64, R_U = 128;
constexpr uint32_t TMEM_COLS = 256;

constexpr uint32_t IDESC_QK = idesc_bf16(128, 64, 0, 0);  // [Q;K] K^T
constexpr uint32_t IDESC_WY = idesc_bf16(128, 64, 1, 0);  // K^T T'^T, V^T T''^T

struct Params {
  const float *g, *beta;
  const int32_t *cu;
  int T, Hqk, Hv;
  int round, rc;  // this launch covers global chunks [round rc, round rc + rc)
  int resident;   // CTAs resident at once (2 per SM): the distance to the next CTA on a slot
  int raw;        // GDN_INPUT_RAW: q, k normalised here, g and beta through -softplus, sigmoid
  const tp::PlanHeader *plan;
  const int32_t *ne_seq, *ne_cs;
  unsigned char *rec;  // this round's records, [rc][Hv]
  int32_t *status;
};

__device__ __forceinline__ uint32_t bar_addr(uint32_t sb, int i) { return sb + OFF_BAR + 8u * i; }

__global__ void __launch_bounds__(NTHREADS, 2)
wy_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const int n_ne = p.plan->n_nonempty, total = p.plan->total_chunks;
  const int g = p.round * p.rc + (int)blockIdx.x;
  if (g >= total) return;
  const int kseq = tp::owner_of_chunk(p.ne_cs, n_ne, g);
  const int n = p.ne_seq[kseq];
  const int t0 = p.cu[n] + (g - p.ne_cs[kseq]) * CH;
  const int Lc = min(CH, p.cu[n + 1] - t0);
  const int j = h / (p.Hv / p.Hqk);
  unsigned char *rec = p.rec + ((size_t)blockIdx.x * p.Hv + h) * tp::REC_BYTES;

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
    // the tiles first: their latency then overlaps the TMEM allocation and
    // the CTA-wide barrier below
    const uint32_t fq = bar_addr(sb, B_QKF), fv = bar_addr(sb, B_VF);
    mbar_arrive_expect_tx(fq, 32768);
    tma_load_3d(sb + OFF_QK + 0, &tm_q, fq, 0, j, t0);
    tma_load_3d(sb + OFF_QK + 8192, &tm_k, fq, 0, j, t0);
    tma_load_3d(sb + OFF_QK + 16384, &tm_q, fq, 64, j, t0);
    tma_load_3d(sb + OFF_QK + 24576, &tm_k, fq, 64, j, t0);
    mbar_arrive_expect_tx(fv, 16384);
    tma_load_3d(sb + OFF_V + 0, &tm_v, fv, 0, h, t0);
    tma_load_3d(sb + OFF_V + 8192, &tm_v, fv, 64, h, t0);
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
    // ------------------------------------------------------------ TMA loads
    if (lane == 0) {
      const uint32_t fq = bar_addr(sb, B_QKF), fv = bar_addr(sb, B_VF);
      // Warm L2 with the tiles of the CTA that will most likely take this
      // slot next (CTAs start in linear order), so that its loads hit L2.
      const int lin = (int)(blockIdx.y * gridDim.x + blockIdx.x) + p.resident;
      if (lin < (int)(gridDim.x * gridDim.y)) {
        const int xn = lin % (int)gridDim.x, hn = lin / (int)gridDim.x;
        const int gn = p.round * p.rc + xn;
        if (gn < total) {
          const int kn = tp::owner_of_chunk(p.ne_cs, n_ne, gn);
          const int tn = p.cu[p.ne_seq[kn]] + (gn - p.ne_cs[kn]) * CH;
          const int jn = hn / (p.Hv / p.Hqk);
          tma_prefetch_3d(&tm_q, 0, jn, tn); tma_prefetch_3d(&tm_q, 64, jn, tn);
          tma_prefetch_3d(&tm_k, 0, jn, tn); tma_prefetch_3d(&tm_k, 64, jn, tn);
          tma_prefetch_3d(&tm_v, 0, hn, tn); tma_prefetch_3d(&tm_v, 64, hn, tn);
        }
      }
      // both tiles land before this CTA can exit
      if (!mbar_wait_landed(fq, 0) || !mbar_wait_landed(fv, 0)) {
        *abort_flag = 1;
        report_status(p.status, GDN_ERR_DEVICE_TIMEOUT);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t dQK = sdesc_sw128(sb + OFF_QK, 16, 1024);             // [Q;K], K-major
      const uint64_t dKmn = sdesc_sw128(sb + OFF_QK + 8192, 16384, 1024);  // K^T, MN-major
      const uint64_t dVmn = sdesc_sw128(sb + OFF_V, 8192, 1024);           // V^T, MN-major
      const uint64_t dTP = sdesc_sw128(sb + OFF_TPH, 16, 1024);            // T', K-major
      const uint64_t dTQ = sdesc_sw128(sb + OFF_TQH, 16, 1024);            // T'', K-major
      bool ok = mbar_wait(bar_addr(sb, B_QKF), 0, abort_flag);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t k16 = ((ks >> 2) * 16384 + (ks & 3) * 32) >> 4;
          mma_bf16(tmem + R_QK, dQK + k16, dQK + (8192 >> 4) + k16, IDESC_QK, ks > 0);
        }
        mma_commit(bar_addr(sb, B_QK));
        ok = mbar_wait(bar_addr(sb, B_T), 0, abort_flag) && mbar_wait(bar_addr(sb, B_VF), 0, abort_flag);
      }
      if (ok) {
        tc_fence_after();
        // W^T = K^T (T'h + T'l)^T ;  U~^T = V^T (T''h + T''l)^T
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t bo = (((ks & 1) ? OFF_TPL - OFF_TPH : 0) + (ks >> 1) * 32) >> 4;
          mma_bf16(tmem + R_W, dKmn + (((ks >> 1) * 2048) >> 4), dTP + bo, IDESC_WY, ks > 0);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t bo = (((ks & 1) ? OFF_TQL - OFF_TQH : 0) + (ks >> 1) * 32) >> 4;
          mma_bf16(tmem + R_U, dVmn + (((ks >> 1) * 2048) >> 4), dTQ + bo, IDESC_WY, ks > 0);
        }
        mma_commit(bar_addr(sb, B_W));
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
    const float gma = exp2f(Ga), gmb = exp2f(Gb);
    const float kda = lane < Lc ? exp2f(GL - Ga) : 0.f;
    const float kdb = lane + 32 < Lc ? exp2f(GL - Gb) : 0.f;
    float *sc = reinterpret_cast<float *>(smem + OFF_SCAL);
    sc[lane] = Ga;        sc[lane + 32] = Gb;
    sc[64 + lane] = gma;  sc[64 + lane + 32] = gmb;
    sc[128 + lane] = kda; sc[128 + lane + 32] = kdb;
    sc[192 + lane] = ba;  sc[192 + lane + 32] = bb;
    sc[256 + lane] = 1.f; sc[256 + lane + 32] = 1.f;  // 1/|q_t|, 1/|k_t|: set by the epilogue
    sc[320 + lane] = 1.f; sc[320 + lane + 32] = 1.f;  // for raw inputs
    float *rs = reinterpret_cast<float *>(rec + tp::REC_SC);
    if (!p.raw) {  // for raw inputs the epilogue writes them with the norms folded in
      rs[lane] = gma;       rs[lane + 32] = gmb;
      rs[64 + lane] = kda;  rs[64 + lane + 32] = kdb;
    }
    if (lane == 0) rs[128] = exp2f(GL);
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_addr(sb, B_SCAL));
  } else if (warp == 3) {
    // the caller's wait limit (a global load kept off the other roles' start)
    if (lane == 0) abort_flag[CTL_LIMIT] = (int)header_wait_limit_us(p.status);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int etid = tid - 128;
    const int half = etid >> 7;   // column half of the 64-column accumulators
    const int row = etid & 127;   // TMEM lane = row of the 128-row tiles
    const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    float *A = reinterpret_cast<float *>(smem + OFF_A);
    float *Tm = reinterpret_cast<float *>(smem + OFF_TM);
    float *Y = reinterpret_cast<float *>(smem + OFF_Y);
    const float *sc = reinterpret_cast<const float *>(smem + OFF_SCAL);
    const float *G2 = sc, *gam = sc + 64, *bet = sc + 192, *rqn = sc + 256, *rkn = sc + 320;
    do {
      if (etid == 0 && !mbar_wait(bar_addr(sb, B_SCAL), 0, abort_flag)) {
        abort_flag[CTL_ABORT] = 1;
        abort_flag[CTL_GROUP] = 1;  // the group's waiter: the next group wait gives up
        report_status(p.status, GDN_ERR_DEVICE_TIMEOUT);
      }
      if (p.raw) {
        // ---- raw inputs: 1/|q_t|, 1/|k_t| from the landed tiles while the first MMA
        // runs.  Thread -> tile row etid / 2 (Q rows, then K rows) and one of its two
        // 128-byte segments (the swizzled order within a segment does not matter to
        // a sum of squares).  The norms are folded into the per-token scalars, not
        // into the bf16 operand tiles: P and A gain 1/|q_t| 1/|k_s| and
        // 1/|k_t| 1/|k_s|, T' gains 1/|k_s|, and the record's e^{G_t} and
        // e^{G_C - G_t} gain 1/|q_t| and 1/|k_t| for the state pass.
        if (!group_wait<NEPI, EPI_BAR>(bar_addr(sb, B_QKF), 0, etid, abort_flag, p.status)) break;
        const int rr = etid >> 1, t = rr & 63;
        const unsigned char *seg = smem + OFF_QK + (rr >> 6) * 8192 + (etid & 1) * 16384 + t * 128;
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 x = *reinterpret_cast<const uint4 *>(seg + 16 * c);
          const uint32_t wd[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float lo = __uint_as_float(wd[i] << 16), hi = __uint_as_float(wd[i] & 0xffff0000u);
            ss = fmaf(lo, lo, fmaf(hi, hi, ss));
          }
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        if ((etid & 1) == 0) {
          const float r = inv_norm(ss);
          float *scw = reinterpret_cast<float *>(smem + OFF_SCAL);
          float *rs = reinterpret_cast<float *>(rec + tp::REC_SC);
          scw[256 + rr] = r;  // 1/|q_t| at [256 + t], 1/|k_t| at [320 + t]
          rs[rr] = sc[64 + rr] * r;  // e^{G_t} / |q_t|, then e^{G_C - G_t} / |k_t|
        }
      }
      if (!group_wait<NEPI, EPI_BAR>(bar_addr(sb, B_QK), 0, etid, abort_flag, p.status)) break;
      // ---- Q K^T -> P (record, hi/lo), K K^T -> A (fp32, shared)
#pragma unroll
      for (int qh = 0; qh < 2; ++qh) {
        float v[16];
        tmem_ld16(tl + R_QK + 32 * half + 16 * qh, v);
        tmem_wait_ld();
        if (row < 64) {
          const int t = row;
          const float Gt = G2[t], rq = rqn[t];
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            float pv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int si = 32 * half + 16 * qh + 8 * q + e;
              pv[e] = (si <= t && t < Lc) ? exp2f(Gt - G2[si]) * v[8 * q + e] * (rq * rkn[si]) : 0.f;
            }
            const uint32_t off = sw128_off(t, 4 * half + 2 * qh + q);
            st_split8(rec + tp::REC_PH + off, rec + tp::REC_PL + off, pv);
          }
        } else {
          const int t = row - 64;
          const float Gt = G2[t], bt = bet[t], rk = rkn[t];
          float *arow = A + t * AST + 32 * half + 16 * qh;
#pragma unroll
          for (int x = 0; x < 16; x += 4) {
            float a[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int si = 32 * half + 16 * qh + x + e;
              a[e] = (si < t && t < Lc) ? bt * exp2f(Gt - G2[si]) * v[x + e] * (rk * rkn[si]) : 0.f;
            }
            *reinterpret_cast<float4 *>(arow + x) = make_float4(a[0], a[1], a[2], a[3]);
          }
        }
      }
      named_bar_sync(EPI_BAR, NEPI);

      // ---- Tm = (I + A)^-1, then T' = Tm diag(beta gamma), T'' = Tm diag(beta), split
      ut_solve<NEPI, EPI_BAR>(A, Tm, Y, etid);
      {
        const int t = etid >> 2, sbeg = 16 * (etid & 3);
        float tp_[16], tq[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float m = (sbeg + e <= t) ? Tm[t * AST + sbeg + e] : 0.f;
          tq[e] = m * bet[sbeg + e];
          tp_[e] = tq[e] * (gam[sbeg + e] * rkn[sbeg + e]);
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint32_t off = sw128_off(t, (sbeg >> 3) + q);
          st_split8(smem + OFF_TPH + off, smem + OFF_TPL + off, tp_ + 8 * q);
          st_split8(smem + OFF_TQH + off, smem + OFF_TQL + off, tq + 8 * q);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(EPI_BAR, NEPI);
      if (etid == 0) mbar_arrive(bar_addr(sb, B_T));

      // ---- W^T -> record (bf16 MN-major image), U~ -> record (fp32 [t][d])
      if (!group_wait<NEPI, EPI_BAR>(bar_addr(sb, B_W), 0, etid, abort_flag, p.status)) break;
      {
        float v[32];
        tmem_ld32(tl + R_W + 32 * half, v);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4 *>(rec + tp::REC_WT + sw128_off(row, 4 * half + q)) = pack_bf16x8(v + 8 * q);
        tmem_ld32(tl + R_U + 32 * half, v);
        tmem_wait_ld();
        float *u = reinterpret_cast<float *>(rec + tp::REC_UT);
#pragma unroll
        for (int x = 0; x < 32; ++x) u[(32 * half + x) * HD + row] = v[x];
      }
    } while (0);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace wy

size_t wy_prep_smem_bytes() { return wy::SMEM_BYTES; }

cudaError_t launch_wy_prep(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                           const float *g, const float *beta, const int32_t *cu, int T, int Hqk,
                           int Hv, int round, int rc, int raw, const void *workspace,
                           const tp::Layout &L, unsigned char *rec, cudaStream_t stream) {
  wy::Params prm;
  prm.g = g; prm.beta = beta; prm.cu = cu; prm.T = T; prm.Hqk = Hqk; prm.Hv = Hv; prm.raw = raw;
  prm.round = round; prm.rc = rc;
  prm.resident = 2 * sm_count();
  unsigned char *ws = static_cast<unsigned char *>(const_cast<void *>(workspace));
  prm.plan = reinterpret_cast<const tp::PlanHeader *>(ws + tp::kPlanHeaderOffset);
  prm.ne_seq = reinterpret_cast<const int32_t *>(ws + L.plan_off);
  prm.ne_cs = prm.ne_seq + L.n_ne_capacity;
  prm.rec = rec;
  prm.status = reinterpret_cast<int32_t *>(ws);
  static std::atomic<bool> smem_set[64];
  cudaError_t e = set_smem_once(wy::wy_prep_kernel, (int)wy::SMEM_BYTES, smem_set);
  if (e != cudaSuccess) return e;
  wy::wy_prep_kernel<<<dim3((unsigned)rc, (unsigned)Hv), wy::NTHREADS, wy::SMEM_BYTES, stream>>>(
      mq, mk, mv, prm);
  return cudaGetLastError();
}

}  // namespace gdn
