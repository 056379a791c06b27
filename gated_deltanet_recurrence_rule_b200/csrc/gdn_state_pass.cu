// gdn_state_pass.cu -- phase 2 of the two-phase tensor-core prefill (the
// inter-chunk state passing), the plan kernel that maps packed sequences to
// global chunks, and the host driver of the two phases.
//
// Per (sequence, value head), chunk after chunk, with the state-free record of
// each chunk already computed by phase 1 (gdn_wy_prep.cu):
//     U^T  = U~^T - S0 W^T                     (M128 N64 K128; U~ added in the epilogue)
//     Oi^T = S0 Q^T,   Oa^T = U^T P^T,   o_t = scale (e^{G_t} Oi_t + Oa_t)
//     dS   = (U diag(e^{G_C - G}))^T K,   S <- e^{G_C} S + dS   (fp32 master copy)
// ("Inside Qwen3.8-27B: Hybrid DeltaNet Architecture, 256k Context, and 24GB
// Local Serving", section "Gated DeltaNet Mechanics": o_t = S_t q_t with the
// fixed-size state kept on chip.)  The state lives in registers of the 512
// epilogue threads (fp32) and as hi + lo bf16 operands in TMEM; only o and
// the final state leave the SM.  The critical path of a chunk is
//     S0 ready -> U MMA -> U epilogue -> dS MMA -> state epilogue -> S0 ready,
// and the output MMAs (Oi, Oa) fill the tensor pipe around it.
//
// Packed sequences are mapped to one list of global chunks (chunks aligned to
// each sequence start).  A workspace that cannot hold every chunk's record is
// used in rounds of RC global chunks: phase 1 then phase 2 per round; the one
// sequence that crosses a round boundary carries its state through the
// workspace.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "gdn_chunk_ops.cuh"
#include "gdn_common.cuh"
#include "gdn_sm100.cuh"
#include "gdn_twophase.cuh"

namespace gdn {

size_t wy_prep_smem_bytes();
cudaError_t launch_wy_prep(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                           const float *g, const float *beta, const int32_t *cu, int T, int Hqk,
                           int Hv, int round, int rc, int raw, const void *workspace,
                           const tp::Layout &L, unsigned char *rec, cudaStream_t stream);

namespace plan {

// One CTA: validates cu_seqlens, lists the non-empty sequences with the first
// global chunk of each (exclusive scan of ceil(L_n / 64)), and writes the
// final state of every empty sequence (= its initial state, or zeros).  Bad
// cu_seqlens set GDN_ERR_BAD_SEQLENS and leave zero chunks to process.
__global__ void __launch_bounds__(1024)
plan_kernel(const int32_t *__restrict__ cu, int N, int T, int Hv, const void *__restrict__ s0,
            void *__restrict__ sfin, size_t state_bytes, tp::PlanHeader *ph, int32_t *ne_seq,
            int32_t *ne_cs, int32_t *status) {
  __shared__ int s_bad, s_run_ne, s_run_ch, s_nempty;
  __shared__ int w_ne[32], w_ch[32];
  __shared__ int s_empty[1024];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) { s_bad = 0; s_run_ne = 0; s_run_ch = 0; }
  __syncthreads();
  for (int i = tid; i <= N; i += blockDim.x) {
    const int c = cu[i];
    bool bad = c < 0 || c > T || (i == 0 && c != 0) || (i == N && c != T);
    if (i < N && cu[i + 1] < c) bad = true;
    if (bad) atomicOr(&s_bad, 1);
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) {
      report_status(status, GDN_ERR_BAD_SEQLENS);
      ph->n_nonempty = 0;
      ph->total_chunks = 0;
    }
    return;
  }
  for (int base = 0; base < N; base += blockDim.x) {
    const int n = base + tid;
    const int L = n < N ? cu[n + 1] - cu[n] : 0;
    const int ne = L > 0 ? 1 : 0, nc = (L + 63) / 64;
    int ie = ne, ic = nc;  // warp-inclusive scans
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int xe = __shfl_up_sync(0xffffffffu, ie, off), xc = __shfl_up_sync(0xffffffffu, ic, off);
      if (lane >= off) { ie += xe; ic += xc; }
    }
    if (lane == 31) { w_ne[wid] = ie; w_ch[wid] = ic; }
    if (tid == 0) s_nempty = 0;
    __syncthreads();
    if (wid == 0) {
      int ve = w_ne[lane], vc = w_ch[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int xe = __shfl_up_sync(0xffffffffu, ve, off), xc = __shfl_up_sync(0xffffffffu, vc, off);
        if (lane >= off) { ve += xe; vc += xc; }
      }
      w_ne[lane] = ve - w_ne[lane];  // exclusive warp offsets
      w_ch[lane] = vc - w_ch[lane];
    }
    __syncthreads();
    const int pe = s_run_ne + w_ne[wid] + ie - ne, pc = s_run_ch + w_ch[wid] + ic - nc;
    if (ne) { ne_seq[pe] = n; ne_cs[pe] = pc; }
    if (n < N && !ne && sfin) s_empty[atomicAdd(&s_nempty, 1)] = n;
    __syncthreads();
    if (tid == blockDim.x - 1) { s_run_ne = pe + ne; s_run_ch = pc + nc; }
    // final state of the empty sequences of this tile = initial state (or 0)
    // (a byte copy: the caller's states are all fp32 or all bf16)
    for (int e = 0; e < s_nempty; ++e) {
      const size_t off = (size_t)s_empty[e] * state_bytes;
      uint4 *dst = reinterpret_cast<uint4 *>(static_cast<unsigned char *>(sfin) + off);
      const uint4 *src =
          s0 ? reinterpret_cast<const uint4 *>(static_cast<const unsigned char *>(s0) + off) : nullptr;
      for (size_t x = tid; x < state_bytes / 16; x += blockDim.x)
        dst[x] = src ? src[x] : make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();
  }
  if (tid == 0) {
    ne_cs[s_run_ne] = s_run_ch;
    ph->n_nonempty = s_run_ne;
    ph->total_chunks = s_run_ch;
  }
}

}  // namespace plan

// One plan_kernel launch (also used by the chunk-form backward, which passes
// dL/dS_final and dL/dS_initial as the initial and final states, so that an
// empty sequence gets dL/dS_initial = dL/dS_final).  state_bytes is one
// sequence's states: Hv x Dv x Dk x element size.
cudaError_t launch_plan(const int32_t *cu, int N, int T, int Hv, const void *s0, void *sfin,
                        size_t state_bytes, tp::PlanHeader *ph, int32_t *ne_seq, int32_t *ne_cs,
                        int32_t *status, cudaStream_t stream) {
  plan::plan_kernel<<<1, 1024, 0, stream>>>(cu, N, T, Hv, s0, sfin, state_bytes, ph, ne_seq, ne_cs,
                                           status);
  return cudaGetLastError();
}

namespace sp {

using namespace sm100;
using namespace chunk;
using tp::CH;
using tp::HD;
using tp::REC_BYTES;

constexpr int NTHREADS = 640;
constexpr int NEPI = 512;   // epilogue threads: 4 column quarters x 128 rows

// ---- shared memory map (bytes) ----
constexpr int NQK = 2, NR = 2;         // ring depths: Q/K tiles, chunk records
constexpr uint32_t QK_STAGE = 32768;   // [Q d0-63 | K d0-63 | Q d64-127 | K d64-127], 64 rows x 128 B each
constexpr uint32_t OFF_QK = 0;
constexpr uint32_t OFF_REC = NQK * QK_STAGE;
constexpr uint32_t OFF_BAR = OFF_REC + NR * REC_BYTES;
constexpr uint32_t OFF_MISC = OFF_BAR + 256;  // [0] TMEM base, [4] control words (chunk::CTL_*), [16] drain mbarrier
constexpr uint32_t SMEM_BYTES = OFF_MISC + 24;
static_assert(OFF_REC % 1024 == 0 && REC_BYTES % 1024 == 0, "alignment");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

enum {
  B_FULL_QK = 0, B_EMPTY_QK = B_FULL_QK + NQK, B_FULL_R = B_EMPTY_QK + NQK, B_EMPTY_R = B_FULL_R + NR,
  // S0 hi / lo written; U ready; U diag(kdec) split written; U split written;
  // dS (and Oi) ready; Oa ready; the outputs of a chunk were read out of TMEM;
  // the MMA issuer's drain
  B_S0H = B_EMPTY_R + NR, B_S0L, B_U, B_UK, B_UO, B_S, B_OA, B_OFREE, B_DRAIN, NBAR
};
static_assert(NBAR * 8 <= 256, "barrier area");

// ---- TMEM columns (128 lanes x 512 columns of 32 bit) ----
constexpr uint32_t R_S = 0;     // 128: U^T - U~^T in [0, 64) (chunk start), then dS (chunk end)
constexpr uint32_t R_OI = 128;  // 64: S0 Q^T
constexpr uint32_t R_OA = 192;  // 64: U^T P^T
// MMA A operands in TMEM (bf16 pairs per column; lane = row of the operand).
constexpr uint32_t T_S0H = 256, T_S0L = 320;  // hi/lo(S0): 128 rows x 128 K
constexpr uint32_t T_UH = 384, T_UL = 416;    // hi/lo(U^T): 128 rows x 64 K
constexpr uint32_t T_UKH = 448, T_UKL = 480;  // hi/lo(U^T diag(kdec))
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t IDESC_SW = idesc_bf16(128, 64, 0, 1, 1);  // -S0 W^T
constexpr uint32_t IDESC_SQ = idesc_bf16(128, 64, 0, 0);     // S0 Q^T, U^T P^T
constexpr uint32_t IDESC_UK = idesc_bf16(128, 128, 0, 1);    // Ukdec^T K

struct Params {
  const int32_t *cu;
  int N, T, Hqk, Hv;
  int round, rc;
  float scale;
  const void *s0;  // caller's initial states, fp32 or (state_bf16) bf16
  void *sfin;      // caller's final states, same type
  int state_bf16;
  void *o;
  const tp::PlanHeader *plan;
  const int32_t *ne_seq, *ne_cs;
  const unsigned char *rec;  // this round's records, [rc][Hv]
  float *carry;              // [2][Hv][128][128]
  int32_t *status;
};

__device__ __forceinline__ uint32_t bar_addr(uint32_t sb, int i) { return sb + OFF_BAR + 8u * i; }

template <typename TO>
__global__ void __launch_bounds__(NTHREADS, 1)
state_pass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const Params p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  // ---- which sequence and which of its chunks this CTA owns in this round
  const int n_ne = p.plan->n_nonempty, total = p.plan->total_chunks;
  const int g_lo = p.round * p.rc, g_hi = min(g_lo + p.rc, total);
  if (g_lo >= g_hi) return;
  const int kseq = tp::owner_of_chunk(p.ne_cs, n_ne, g_lo) + (int)blockIdx.x;
  if (kseq >= n_ne) return;
  const int cs = p.ne_cs[kseq], ce = p.ne_cs[kseq + 1];
  if (cs >= g_hi) return;
  const int ga = max(cs, g_lo), gb = min(ce, g_hi);
  const int nch = gb - ga;
  const int n = p.ne_seq[kseq];
  const int j = h / (p.Hv / p.Hqk);
  const int seq_begin = p.cu[n], seq_end = p.cu[n + 1];
  const size_t hstate = (size_t)HD * HD;
  const size_t sbase = ((size_t)n * p.Hv + h) * hstate;
  // the state comes from the caller (first chunk of the sequence) or from the
  // carry of the previous round, and goes to the caller or to the carry
  const int ueb = p.state_bf16 ? 2 : 4;  // bytes per element of the caller's states
  const bool src_bf16 = (ga == cs) && p.state_bf16, dst_bf16 = (gb == ce) && p.state_bf16;
  const void *src = (ga == cs)
      ? (p.s0 ? static_cast<const void *>(static_cast<const unsigned char *>(p.s0) + sbase * ueb) : nullptr)
      : static_cast<const void *>(p.carry + ((size_t)((p.round - 1) & 1) * p.Hv + h) * hstate);
  void *dst = (gb == ce)
      ? (p.sfin ? static_cast<void *>(static_cast<unsigned char *>(p.sfin) + sbase * ueb) : nullptr)
      : static_cast<void *>(p.carry + ((size_t)(p.round & 1) * p.Hv + h) * hstate);

  const uint32_t sb = smem_addr(smem);
  if (sb & 1023u) {  // swizzled operand tiles need 1024-byte alignment
    if (tid == 0) report_status(p.status, GDN_ERR_UNSUPPORTED);
    return;
  }
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
  if (tid == 0) {
    for (int i = 0; i < NBAR; ++i) mbar_init(bar_addr(sb, i), 1);
    // barriers the 16 epilogue warps arrive on, one arrival per warp
    for (int b : {(int)B_S0H, (int)B_S0L, (int)B_UK, (int)B_UO, (int)B_OFREE})
      mbar_init(bar_addr(sb, b), NEPI / 32);
    // a record slot is free once its MMAs completed AND every epilogue warp read it
    for (int i = 0; i < NR; ++i) mbar_init(bar_addr(sb, B_EMPTY_R + i), 1 + NEPI / 32);
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
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      constexpr int PF = 4;  // L2 prefetch distance in chunks
      auto chunk_t0 = [&](int c) { return seq_begin + (ga - cs + c) * CH; };
      auto chunk_rec = [&](int c) {
        return p.rec + ((size_t)(ga + c - g_lo) * p.Hv + h) * REC_BYTES;
      };
      for (int c = 0; c < PF && c < nch; ++c) {
        const int t = chunk_t0(c);
        tma_prefetch_3d(&tm_q, 0, j, t); tma_prefetch_3d(&tm_q, 64, j, t);
        tma_prefetch_3d(&tm_k, 0, j, t); tma_prefetch_3d(&tm_k, 64, j, t);
        bulk_prefetch_l2(chunk_rec(c), REC_BYTES);
      }
      int issued_qk = 0, issued_r = 0;
      for (int c = 0; c < nch; ++c) {
        const int s = c % NQK, sr = c % NR;
        const int t0 = chunk_t0(c);
        if (c + PF < nch) {
          const int t = chunk_t0(c + PF);
          tma_prefetch_3d(&tm_q, 0, j, t); tma_prefetch_3d(&tm_q, 64, j, t);
          tma_prefetch_3d(&tm_k, 0, j, t); tma_prefetch_3d(&tm_k, 64, j, t);
          bulk_prefetch_l2(chunk_rec(c + PF), REC_BYTES);
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
        if (!mbar_wait(bar_addr(sb, B_EMPTY_R + sr), ((c / NR) & 1) ^ 1, abort_flag)) break;
        const uint32_t fr = bar_addr(sb, B_FULL_R + sr);
        mbar_arrive_expect_tx(fr, REC_BYTES);
        bulk_load(sb + OFF_REC + sr * REC_BYTES, chunk_rec(c), REC_BYTES, fr);
        issued_r = c + 1;
      }
      if (issued_qk < nch || issued_r < nch) {
        *abort_flag = 1;
        report_status(p.status, GDN_ERR_DEVICE_TIMEOUT);
      }
      // Every load this thread issued lands before the CTA can exit (each
      // buffer's latest fill; earlier fills were consumed before it was issued).
      for (int c = max(issued_qk - NQK, 0); c < issued_qk; ++c)
        mbar_wait_landed(bar_addr(sb, B_FULL_QK + c % NQK), (c / NQK) & 1, 50000000ull);
      for (int c = max(issued_r - NR, 0); c < issued_r; ++c)
        mbar_wait_landed(bar_addr(sb, B_FULL_R + c % NR), (c / NR) & 1, 50000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // A converged warp: lane 0 waits, one elected lane issues each group of
    // MMAs and its commits (far fewer issue cycles than a lone diverged lane).
    // Order per chunk: U (chain), Oi (runs while the epilogue splits U), dS
    // (chain), Oa (runs while the epilogue updates the state).
    const uint64_t dQK0 = sdesc_sw128(sb + OFF_QK, 16, 1024);            // Q, K-major
    const uint64_t dKmn0 = sdesc_sw128(sb + OFF_QK + 8192, 16384, 1024); // K as MN-major operand
    const uint64_t dW0 = sdesc_sw128(sb + OFF_REC + tp::REC_WT, 8192, 1024);  // W^T, MN-major
    const uint64_t dP0 = sdesc_sw128(sb + OFF_REC + tp::REC_PH, 16, 1024);    // P hi / lo, K-major
    auto wait = [&](int b, uint32_t parity) {
      int ok = 1;
      if (lane == 0) ok = mbar_wait(bar_addr(sb, b), parity, abort_flag);
      return __shfl_sync(0xffffffffu, ok, 0) != 0;
    };
    bool ok = true;
    for (int c = 0; c < nch && ok; ++c) {
      const int s = c % NQK, sr = c % NR;
      const uint32_t ph = c & 1;
      const uint64_t dQK = dQK0 + s * (QK_STAGE >> 4), dKmn = dKmn0 + s * (QK_STAGE >> 4);
      const uint64_t dW = dW0 + sr * (REC_BYTES >> 4), dP = dP0 + sr * (REC_BYTES >> 4);
      // U^T - U~^T = -S0h W^T   (S0 hi from TMEM)
      if (!(ok = wait(B_FULL_R + sr, (c / NR) & 1) && wait(B_S0H, ph))) break;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ts(tmem + R_S, tmem + T_S0H + 8 * ks, dW + ((ks * 2048) >> 4), IDESC_SW, ks > 0);
        mma_commit(bar_addr(sb, B_U));
      }
      __syncwarp();
      // Oi^T = (S0h + S0l) Q^T, once S0 is complete and the previous outputs were read
      if (!(ok = wait(B_FULL_QK + s, (c / NQK) & 1) && wait(B_S0L, ph) &&
                 (c == 0 || wait(B_OFREE, (c - 1) & 1))))
        break;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int ks = 0; ks < 16; ++ks) {
          const int k = ks >> 1;
          const uint32_t k16 = ((k >> 2) * 16384 + (k & 3) * 32) >> 4;
          mma_bf16_ts(tmem + R_OI, tmem + ((ks & 1) ? T_S0L : T_S0H) + 8 * k, dQK + k16, IDESC_SQ,
                      ks > 0);
        }
      }
      __syncwarp();
      // dS = (Ukh + Ukl)^T K   (U diag(kdec) from TMEM)
      if (!(ok = wait(B_UK, ph))) break;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const int kk = ks >> 1;
          mma_bf16_ts(tmem + R_S, tmem + ((ks & 1) ? T_UKL : T_UKH) + 8 * kk,
                      dKmn + ((kk * 2048) >> 4), IDESC_UK, ks > 0);
        }
        mma_commit(bar_addr(sb, B_S));
      }
      __syncwarp();
      // Oa^T = Uh Ph^T + Ul Ph^T + Uh Pl^T   (U from TMEM)
      if (!(ok = wait(B_UO, ph))) break;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int ks = 0; ks < 12; ++ks) {
          const int part = ks % 3, kk = ks / 3;  // (Uh,Ph), (Ul,Ph), (Uh,Pl)
          const uint32_t bo = ((part == 2 ? tp::REC_PL - tp::REC_PH : 0) + kk * 32) >> 4;
          mma_bf16_ts(tmem + R_OA, tmem + (part == 1 ? T_UL : T_UH) + 8 * kk, dP + bo, IDESC_SQ,
                      ks > 0);
        }
        mma_commit(bar_addr(sb, B_OA));
        mma_commit(bar_addr(sb, B_EMPTY_QK + s));
        mma_commit(bar_addr(sb, B_EMPTY_R + sr));
      }
      __syncwarp();
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      report_status(p.status, GDN_ERR_DEVICE_TIMEOUT);
    }
    // Drain: every MMA this warp issued finishes before TMEM is freed.
    if (elect_one()) {
      mma_commit(bar_addr(sb, B_DRAIN));
      mbar_wait_landed(bar_addr(sb, B_DRAIN), 0, 50000000ull);
    }
    __syncwarp();
  } else if (warp == 3) {
    // the caller's wait limit (a global load kept off the other roles' start)
    if (lane == 0) abort_flag[CTL_LIMIT] = (int)header_wait_limit_us(p.status);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    // 16 warps, each on its own: a warp waits for an MMA group through its
    // lane 0 and signals the MMA issuer by one arrival per warp (the barriers
    // the issuer waits on count 16), so no barrier spans the epilogue warps
    // and a slow warp delays only the MMAs that need its columns.
    const int etid = tid - 128;
    const int ewq = etid >> 7;   // column quarter
    const int row = etid & 127;  // TMEM lane = row (Dv index) of the 128-row tiles
    const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    auto warp_wait = [&](int b, uint32_t parity) {
      int ok = 1;
      if (lane == 0 && !(ok = mbar_wait(bar_addr(sb, b), parity, abort_flag))) {
        abort_flag[CTL_ABORT] = 1;
        report_status(p.status, GDN_ERR_DEVICE_TIMEOUT);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok) tc_fence_after();
      return ok != 0;
    };
    // after this warp's tcgen05.st have completed (tmem_wait_st)
    auto warp_signal = [&](int b) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_addr(sb, b));
    };

    // fp32 master state: row `row`, columns [32 ewq, 32 ewq + 32); S0 = hi + lo in TMEM
    float S[32];
    {
      const size_t e0 = (size_t)row * HD + 32 * ewq;
#pragma unroll
      for (int x = 0; x < 32; x += 4) {
        if (src) load_state4(src, e0 + x, src_bf16, S + x);
        else S[x] = S[x + 1] = S[x + 2] = S[x + 3] = 0.f;
      }
      uint32_t hw[16], lw[16];
      split_words<16>(S, hw, lw);
      tmem_st16(tl + T_S0H + 16 * ewq, hw);
      tmem_st16(tl + T_S0L + 16 * ewq, lw);
      tmem_wait_st();
    }
    warp_signal(B_S0H);
    warp_signal(B_S0L);

    // U~ of the chunk about to run, read from its record while the previous
    // chunk's dS product runs
    float un[16];
    auto fetch_ut = [&](int c) {
      const int sr = c % NR;
      if (!warp_wait(B_FULL_R + sr, (c / NR) & 1)) return false;
      const float *ut = reinterpret_cast<const float *>(smem + OFF_REC + sr * REC_BYTES + tp::REC_UT) + row;
#pragma unroll
      for (int x = 0; x < 16; ++x) un[x] = ut[(16 * ewq + x) * HD];
      return true;
    };
    // The outputs of chunk c leave TMEM at the end of chunk c and go to HBM
    // during chunk c + 1, a quarter at each of its four waits, so that the
    // store path drains in the background.
    float out[16];
    int out_t0 = 0, out_n = 0;  // this thread's first token of the chunk whose outputs `out`
                                // holds, and how many of its 16 tokens that chunk has
    auto store_out = [&](int part) {
      TO *op = static_cast<TO *>(p.o) + ((size_t)out_t0 * p.Hv + h) * HD + row;
#pragma unroll
      for (int x = 4 * part; x < 4 * part + 4; ++x)
        if (x < out_n) op[(size_t)x * p.Hv * HD] = from_f32<TO>(out[x]);
    };
    bool ok = fetch_ut(0);
    for (int c = 0; c < nch && ok; ++c) {
      const int sr = c % NR;
      const uint32_t ph = c & 1;
      const int t0 = seq_begin + (ga - cs + c) * CH;
      const int Lc = min(CH, seq_end - t0);
      const float *gam = reinterpret_cast<const float *>(smem + OFF_REC + sr * REC_BYTES + tp::REC_SC);
      const float *kdec = gam + 64;

      // ---- U = (U - U~) + U~ -> hi/lo(U^T diag(kdec)) for dS first, then hi/lo(U^T) for Oa
      if (!(ok = warp_wait(B_U, ph))) break;
      {
        float v[16];
        tmem_ld16(tl + R_S + 16 * ewq, v);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 16; x += 2) {
          const float2 a = __fadd2_rn(make_float2(v[x], v[x + 1]), make_float2(un[x], un[x + 1]));
          v[x] = a.x; v[x + 1] = a.y;
        }
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {
          const float4 ka = *reinterpret_cast<const float4 *>(kdec + 16 * ewq + 8 * hq);
          const float4 kb = *reinterpret_cast<const float4 *>(kdec + 16 * ewq + 8 * hq + 4);
          const float2 w0 = __fmul2_rn(make_float2(v[8 * hq + 0], v[8 * hq + 1]), make_float2(ka.x, ka.y));
          const float2 w1 = __fmul2_rn(make_float2(v[8 * hq + 2], v[8 * hq + 3]), make_float2(ka.z, ka.w));
          const float2 w2 = __fmul2_rn(make_float2(v[8 * hq + 4], v[8 * hq + 5]), make_float2(kb.x, kb.y));
          const float2 w3 = __fmul2_rn(make_float2(v[8 * hq + 6], v[8 * hq + 7]), make_float2(kb.z, kb.w));
          const float w[8] = {w0.x, w0.y, w1.x, w1.y, w2.x, w2.y, w3.x, w3.y};
          uint32_t hw[4], lw[4];
          split_words<4>(w, hw, lw);
          tmem_st4(tl + T_UKH + 8 * ewq + 4 * hq, hw);
          tmem_st4(tl + T_UKL + 8 * ewq + 4 * hq, lw);
        }
        tmem_wait_st();
        warp_signal(B_UK);
        store_out(0);
        uint32_t hw[8], lw[8];
        split_words<8>(v, hw, lw);
        tmem_st8(tl + T_UH + 8 * ewq, hw);
        tmem_st8(tl + T_UL + 8 * ewq, lw);
        tmem_wait_st();
      }
      warp_signal(B_UO);
      store_out(1);

      // ---- state: S = gamma_C S + dS (fp32); hi(S) first (the next U product), then lo(S)
      if (!(ok = warp_wait(B_S, ph))) break;
      {
        const float gC = gam[128];
        const float2 g2 = make_float2(gC, gC);
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {
          float v[16];
          tmem_ld16(tl + R_S + 32 * ewq + 16 * hq, v);
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 16; x += 2) {
            const float2 a = __ffma2_rn(g2, make_float2(S[16 * hq + x], S[16 * hq + x + 1]),
                                        make_float2(v[x], v[x + 1]));
            S[16 * hq + x] = a.x; S[16 * hq + x + 1] = a.y;
          }
          uint32_t hw[8];
          hi_words<8>(S + 16 * hq, hw);
          tmem_st8(tl + T_S0H + 16 * ewq + 8 * hq, hw);
        }
        tmem_wait_st();
      }
      warp_signal(B_S0H);
      store_out(2);
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {
        uint32_t lw[8];
        lo_words<8>(S + 16 * hq, lw);
        tmem_st8(tl + T_S0L + 16 * ewq + 8 * hq, lw);
      }
      tmem_wait_st();
      warp_signal(B_S0L);
      store_out(3);

      // ---- outputs o_t = scale (e^{G_t} Oi_t + Oa_t) out of TMEM
      if (!(ok = warp_wait(B_OA, ph))) break;
      {
        float va[16];
        tmem_ld16(tl + R_OI + 16 * ewq, out);
        tmem_ld16(tl + R_OA + 16 * ewq, va);
        tmem_wait_ld();
        const float2 sc2 = make_float2(p.scale, p.scale);
#pragma unroll
        for (int x = 0; x < 16; x += 4) {
          const float4 g4 = *reinterpret_cast<const float4 *>(gam + 16 * ewq + x);
          const float2 a = __ffma2_rn(make_float2(g4.x, g4.y), make_float2(out[x], out[x + 1]),
                                      make_float2(va[x], va[x + 1]));
          const float2 b = __ffma2_rn(make_float2(g4.z, g4.w), make_float2(out[x + 2], out[x + 3]),
                                      make_float2(va[x + 2], va[x + 3]));
          const float2 a2 = __fmul2_rn(sc2, a), b2 = __fmul2_rn(sc2, b);
          out[x] = a2.x; out[x + 1] = a2.y; out[x + 2] = b2.x; out[x + 3] = b2.y;
        }
      }
      out_t0 = t0 + 16 * ewq;
      out_n = min(16, Lc - 16 * ewq);
      warp_signal(B_OFREE);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_addr(sb, B_EMPTY_R + sr));  // this warp is done with the record
      // ---- the next chunk's U~, while its U product runs
      if (c + 1 < nch && !(ok = fetch_ut(c + 1))) break;
    }
    if (ok && abort_flag[CTL_ABORT] == 0) {
#pragma unroll
      for (int part = 0; part < 4; ++part) store_out(part);
      if (dst) {
        const size_t e0 = (size_t)row * HD + 32 * ewq;
#pragma unroll
        for (int x = 0; x < 32; x += 4) store_state4(dst, e0 + x, dst_bf16, S + x);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace sp

// ---------------------------------------------------------------- host side

using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                              const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                              const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeFn encode_fn() {
  static std::atomic<EncodeFn> fn{nullptr};
  EncodeFn f = fn.load(std::memory_order_acquire);
  if (!f) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      f = reinterpret_cast<EncodeFn>(ptr);
      fn.store(f, std::memory_order_release);
    }
  }
  return f;
}

bool make_qkv_map(CUtensorMap *m, const void *base, int H, int T) {
  EncodeFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)tp::HD, (cuuint64_t)H, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)tp::HD * 2, (cuuint64_t)H * tp::HD * 2};
  const cuuint32_t box[3] = {64, 1, tp::CH};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Rounds of the pipelined schedule: about kPipeRounds rounds of at least
// kMinRoundChunks global chunks each, records double-buffered.
constexpr int64_t kPipeRounds = 6, kMinRoundChunks = 8;

static int64_t pipelined_round_chunks(int64_t N, int64_t T) {
  const int64_t bound = tp::chunk_bound(N, T);
  return std::max<int64_t>(kMinRoundChunks, (bound + kPipeRounds - 1) / kPipeRounds);
}

size_t twophase_workspace_bytes(int64_t N, int64_t T, int Hv) {
  const tp::Layout L = tp::layout(N, Hv);
  return L.fixed + 2 * (size_t)pipelined_round_chunks(N, T) * L.rec_row;
}

size_t twophase_min_workspace_bytes(int64_t N, int Hv) {
  const tp::Layout L = tp::layout(N, Hv);
  return L.fixed + L.rec_row;
}

size_t twophase_round_workspace_bytes(int64_t N, int Hv, int64_t chunks_per_round) {
  const tp::Layout L = tp::layout(N, Hv);
  return L.fixed + (size_t)chunks_per_round * L.rec_row;
}

// Kernel launches of one two-phase prefill with this workspace: the plan
// kernel, then phase 1 and phase 2 per round.
int64_t twophase_launch_count(int64_t N, int64_t T, int Hv, size_t workspace_bytes) {
  if (T == 0) return 1;
  const tp::Layout L = tp::layout(N, Hv);
  const int64_t bound = tp::chunk_bound(N, T);
  const bool pipelined = workspace_bytes >= twophase_workspace_bytes(N, T, Hv);
  const int64_t fit = (int64_t)((workspace_bytes - L.fixed) / L.rec_row);
  const int64_t rc = std::min<int64_t>(pipelined ? pipelined_round_chunks(N, T) : std::min(bound, fit), 1 << 20);
  return 1 + 2 * ((bound + rc - 1) / rc);
}

template <typename TO>
static cudaError_t launch_state_pass(const CUtensorMap &mq, const CUtensorMap &mk,
                                     const sp::Params &prm, int grid_x, cudaStream_t stream) {
  auto kern = sp::state_pass_kernel<TO>;
  static std::atomic<bool> smem_set[64];
  cudaError_t e = set_smem_once(kern, (int)sp::SMEM_BYTES, smem_set);
  if (e != cudaSuccess) return e;
  kern<<<dim3((unsigned)grid_x, (unsigned)prm.Hv), sp::NTHREADS, sp::SMEM_BYTES, stream>>>(mq, mk, prm);
  return cudaGetLastError();
}

// Internal streams and events of the pipelined schedule: phase 1 runs on
// `prep`, phase 2 on `chain` (higher priority, so its CTAs get the SMs that
// free up first).  One pair per (device, caller stream), for up to
// kPairsPerDevice caller streams per device, created by the first pipelined
// prefill issued on that caller stream and kept until the process exits, so
// prefills issued on different caller streams do not queue behind one
// another.  Further caller streams share the device's first pair (their
// prefills are then ordered after one another, which is correct but not
// concurrent).
namespace {
constexpr int kMaxDevices = 64, kEventRing = 4, kPairsPerDevice = 8;
struct DeviceStreams {
  bool ready = false;
  cudaStream_t owner = nullptr;  // the caller stream this pair serves
  cudaStream_t prep = nullptr, chain = nullptr;
  cudaEvent_t start = nullptr, prep_done = nullptr, ev_p[kEventRing] = {}, ev_c[kEventRing] = {};
};
std::mutex g_streams_mutex;
DeviceStreams g_streams[kMaxDevices][kPairsPerDevice];

cudaError_t device_streams(cudaStream_t caller, DeviceStreams **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  int slot = 0;  // the caller's pair, else the first free one, else the shared first one
  for (int i = 0; i < kPairsPerDevice; ++i) {
    if (g_streams[dev][i].ready && g_streams[dev][i].owner == caller) { slot = i; break; }
    if (!g_streams[dev][i].ready) { slot = i; break; }
  }
  DeviceStreams &d = g_streams[dev][slot];
  if (!d.ready) {
    d.owner = caller;
    int least = 0, greatest = 0;
    if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithPriority(&d.prep, cudaStreamNonBlocking, least)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithPriority(&d.chain, cudaStreamNonBlocking, greatest)) != cudaSuccess) return e;
    cudaEvent_t *all[] = {&d.start, &d.prep_done};
    for (cudaEvent_t *ev : all)
      if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return e;
    for (int i = 0; i < kEventRing; ++i) {
      if ((e = cudaEventCreateWithFlags(&d.ev_p[i], cudaEventDisableTiming)) != cudaSuccess) return e;
      if ((e = cudaEventCreateWithFlags(&d.ev_c[i], cudaEventDisableTiming)) != cudaSuccess) return e;
    }
    d.ready = true;
  }
  *out = &d;
  return cudaSuccess;
}
}  // namespace

// Plan, then per round: phase 1 (WY prep of every chunk of the round) and
// phase 2 (state passing).  With a workspace of twophase_workspace_bytes or
// more, rounds are pipelined: phase 1 of round r + 1 runs on the SMs phase 2
// of round r leaves free, each round's records still in L2 when phase 2 reads
// them (two record buffers).  With less (>= twophase_min_workspace_bytes) the
// rounds run one after another on `stream` with as many chunks as fit.
cudaError_t launch_prefill_twophase(const void *q, const void *k, const void *v, const float *g,
                                    const float *beta, const int32_t *cu, int N, long long T_,
                                    int Hqk, int Hv, int o_dtype, int state_dtype, int input_form,
                                    float scale, const void *s0, void *sfin, void *o,
                                    void *workspace, size_t workspace_bytes, cudaStream_t stream) {
  const int T = (int)T_;
  const int raw = input_form == GDN_INPUT_RAW;
  const tp::Layout L = tp::layout(N, Hv);
  unsigned char *ws = static_cast<unsigned char *>(workspace);
  int32_t *status = reinterpret_cast<int32_t *>(ws);
  tp::PlanHeader *ph = reinterpret_cast<tp::PlanHeader *>(ws + tp::kPlanHeaderOffset);
  int32_t *ne_seq = reinterpret_cast<int32_t *>(ws + L.plan_off);
  int32_t *ne_cs = ne_seq + L.n_ne_capacity;

  CUtensorMap mq, mk, mv;
  if (T > 0 && (!make_qkv_map(&mq, q, Hqk, T) || !make_qkv_map(&mk, k, Hqk, T) ||
                !make_qkv_map(&mv, v, Hv, T)))
    return cudaErrorInvalidValue;
  const int64_t bound = tp::chunk_bound(N, T);
  const bool pipelined = workspace_bytes >= twophase_workspace_bytes(N, T, Hv);
  const int64_t fit = (int64_t)((workspace_bytes - L.fixed) / L.rec_row);
  const int rc = (int)std::min<int64_t>(
      pipelined ? pipelined_round_chunks(N, T) : std::min<int64_t>(bound, fit), 1 << 20);
  const int rounds = (int)((bound + rc - 1) / rc);

  sp::Params prm;
  prm.cu = cu; prm.N = N; prm.T = T; prm.Hqk = Hqk; prm.Hv = Hv; prm.rc = rc; prm.scale = scale;
  prm.s0 = s0; prm.sfin = sfin; prm.state_bf16 = state_dtype == GDN_DTYPE_BF16; prm.o = o;
  const size_t state_bytes = (size_t)Hv * 128 * 128 * (prm.state_bf16 ? 2 : 4);
  prm.plan = ph; prm.ne_seq = ne_seq; prm.ne_cs = ne_cs;
  prm.carry = reinterpret_cast<float *>(ws + L.carry_off);
  prm.status = status;
  const int grid_x = std::min(N, rc);
  auto state_pass = [&](cudaStream_t st) {
    return (o_dtype == GDN_DTYPE_BF16) ? launch_state_pass<__nv_bfloat16>(mq, mk, prm, grid_x, st)
                                       : launch_state_pass<float>(mq, mk, prm, grid_x, st);
  };
  cudaError_t e;

  if (!pipelined) {
    plan::plan_kernel<<<1, 1024, 0, stream>>>(cu, N, T, Hv, s0, sfin, state_bytes, ph, ne_seq,
                                             ne_cs, status);
    if ((e = cudaGetLastError()) != cudaSuccess || T == 0) return e;
    prm.rec = ws + L.rec_off;
    for (int r = 0; r < rounds; ++r) {
      e = launch_wy_prep(mq, mk, mv, g, beta, cu, T, Hqk, Hv, r, rc, raw, workspace, L, ws + L.rec_off,
                         stream);
      if (e != cudaSuccess) return e;
      prm.round = r;
      if ((e = state_pass(stream)) != cudaSuccess) return e;
    }
    return cudaSuccess;
  }

  // Pipelined rounds on the device's two internal streams, joined to `stream`
  // by events (this also works while `stream` is being captured into a graph).
  std::lock_guard<std::mutex> lock(g_streams_mutex);
  DeviceStreams *d = nullptr;
  if ((e = device_streams(stream, &d)) != cudaSuccess) return e;
  if ((e = cudaEventRecord(d->start, stream)) != cudaSuccess) return e;
  if ((e = cudaStreamWaitEvent(d->prep, d->start, 0)) != cudaSuccess) return e;
  if ((e = cudaStreamWaitEvent(d->chain, d->start, 0)) != cudaSuccess) return e;
  plan::plan_kernel<<<1, 1024, 0, d->prep>>>(cu, N, T, Hv, s0, sfin, state_bytes, ph, ne_seq,
                                             ne_cs, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (T == 0) {
    if ((e = cudaEventRecord(d->prep_done, d->prep)) != cudaSuccess) return e;
    return cudaStreamWaitEvent(stream, d->prep_done, 0);
  }
  for (int r = 0; r < rounds; ++r) {
    unsigned char *rec = ws + L.rec_off + (size_t)(r & 1) * rc * L.rec_row;
    // phase 1 of round r reuses the buffer phase 2 of round r - 2 read
    if (r >= 2 && (e = cudaStreamWaitEvent(d->prep, d->ev_c[(r - 2) % kEventRing], 0)) != cudaSuccess)
      return e;
    e = launch_wy_prep(mq, mk, mv, g, beta, cu, T, Hqk, Hv, r, rc, raw, workspace, L, rec, d->prep);
    if (e != cudaSuccess) return e;
    if ((e = cudaEventRecord(d->ev_p[r % kEventRing], d->prep)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(d->chain, d->ev_p[r % kEventRing], 0)) != cudaSuccess) return e;
    prm.round = r;
    prm.rec = rec;
    if ((e = state_pass(d->chain)) != cudaSuccess) return e;
    if ((e = cudaEventRecord(d->ev_c[r % kEventRing], d->chain)) != cudaSuccess) return e;
  }
  // phase 2 of the last round follows every earlier launch of both streams
  return cudaStreamWaitEvent(stream, d->ev_c[(rounds - 1) % kEventRing], 0);
}

}  // namespace gdn
