// gdn_twophase.cuh -- layouts shared by the two-phase tensor-core prefill:
// the per-chunk record that the WY-prep kernel writes and the state-pass
// kernel reads, the workspace map, and the chunk lookup over packed sequences.
//
// Chunked form of the gated delta rule ("Inside Qwen3.8-27B: Hybrid DeltaNet
// Architecture, 256k Context, and 24GB Local Serving", section "Gated DeltaNet
// Mechanics": prefill runs in a block-parallel form, decode token by token).
// For a chunk of C = 64 tokens with start state S0 and local log-decay prefix
// sums G_t:
//     A_ts = beta_t e^{G_t - G_s} k_t.k_s  (s < t),     Tm = (I + A)^-1
//     W  = Tm diag(beta e^G) K,   U~ = Tm diag(beta) V          (state-free)
//     P_ts = e^{G_t - G_s} q_t.k_s  (s <= t)                    (state-free)
//     U  = U~ - W S0^T
//     O  = diag(e^G) Q S0^T + P U
//     S  = e^{G_C} S0 + U^T diag(e^{G_C - G}) K
// Phase 1 computes everything marked state-free for every (chunk, value head)
// at once; phase 2 walks the chunks of each (sequence, value head) in order
// and does only the three state-dependent products.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "gdn_common.cuh"

namespace gdn {
namespace tp {

constexpr int CH = 64;   // chunk length
constexpr int HD = 128;  // head dim (Dk = Dv)

// ---- per-(chunk, value head) record, 1024-byte aligned pieces ----
// The bf16 tiles are byte images of 128-byte-swizzled shared-memory operand
// tiles (swizzle phase taken from the row index), so one bulk copy to a
// 1024-byte aligned shared address yields MMA-ready operands.
constexpr uint32_t REC_WT = 0;       // W^T bf16, MN-major: 128 rows (d) x 64 t
constexpr uint32_t REC_PH = 16384;   // hi(P) bf16, K-major: 64 rows (t) x 64 s
constexpr uint32_t REC_PL = 24576;   // lo(P) = bf16(P - hi(P))
constexpr uint32_t REC_UT = 32768;   // U~ fp32 [64 t][128 d], row-major
constexpr uint32_t REC_SC = 65536;   // fp32: gamma_t = e^{G_t} [64], kdec_t = e^{G_C - G_t} [64], e^{G_C}
constexpr uint32_t REC_BYTES = 66560;
static_assert(REC_BYTES % 1024 == 0, "records keep 1024-byte alignment");

// ---- workspace map ----
// [0, 256)           WorkspaceHeader (status word) + plan scalars
// [plan, +)          ne_seq[N] (ids of the non-empty sequences, in order),
//                    ne_cs[N + 1] (first global chunk of each, then the total)
// [carry, +)         2 x Hv x 128 x 128 fp32: the state of the one sequence
//                    that crosses a round boundary (alternating by round)
// [rec, +)           RC x Hv records (one round of RC global chunks)
struct PlanHeader {  // lives at byte 16 of the workspace header
  int32_t n_nonempty;
  int32_t total_chunks;
};
constexpr size_t kPlanHeaderOffset = 16;

struct Layout {
  size_t plan_off, carry_off, rec_off, fixed, rec_row;  // rec_row = Hv x REC_BYTES
  int64_t n_ne_capacity;                                // N: ne_cs starts at ne_seq + N
};

__host__ __device__ inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ inline Layout layout(int64_t N, int64_t Hv) {
  Layout L;
  L.n_ne_capacity = N;
  L.plan_off = kWorkspaceHeaderBytes;
  L.carry_off = round_up(L.plan_off + sizeof(int32_t) * (2 * (size_t)N + 1), 1024);
  L.rec_off = round_up(L.carry_off + 2 * (size_t)Hv * HD * HD * sizeof(float), 1024);
  L.fixed = L.rec_off;
  L.rec_row = (size_t)Hv * REC_BYTES;
  return L;
}

// Upper bound on the number of chunks of N sequences holding T tokens in all
// (every sequence adds at most one partial chunk).
__host__ inline int64_t chunk_bound(int64_t N, int64_t T) { return (T + CH - 1) / CH + N; }

// Index k of the non-empty sequence that owns global chunk g: the last k with
// ne_cs[k] <= g (binary search; 0 <= g < total chunks).
__device__ __forceinline__ int owner_of_chunk(const int32_t *__restrict__ ne_cs, int n_ne, int g) {
  int lo = 0, hi = n_ne - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ne_cs[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace tp

// Tensor map of a packed [T, H, 128] bf16 tensor viewed as (d, head, token),
// box 64 d x 1 head x 64 tokens, 128-byte swizzle: one 64 x 64 operand half
// per load.  Tokens past T read as zeros.
bool make_qkv_map(CUtensorMap *m, const void *base, int H, int T);

}  // namespace gdn
