// gdn_chunk_ops.cuh -- per-chunk building blocks shared by the tensor-core
// prefill kernels: the fp32 unit lower-triangular inverse Tm = (I + A)^-1 of
// the 64 x 64 chunk system (the UT transform of the WY representation), and
// the conversions of fp32 values into bf16 hi/lo operand pairs.
#pragma once

#include <stdint.h>

#include "gdn_common.cuh"
#include "gdn_sm100.cuh"

namespace gdn {
namespace chunk {

using namespace sm100;

constexpr int AST = 68;  // fp32 row stride of A and Tm in shared memory (conflict-free float4 rows)

// ---- warp-level m16n8k8 tf32 MMAs with a 3-term split (x = hi + lo, hi =
// tf32(x)): hi*hi + hi*lo + lo*hi carries ~fp32 accuracy.
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void mma_tf32_16x8x8(float *d, const uint32_t *a, const uint32_t *b) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// D (16x8 fp32, fragment layout) = X (16 x 8 KS, row-major, stride ldx) *
// Y (8 KS x 8, row-major, stride ldy), with the 3-term split.
template <int KS>
__device__ __forceinline__ void mma3_16x8(float *d, const float *X, int ldx, const float *Y, int ldy,
                                          int lane) {
  const int gid = lane >> 2, tig = lane & 3;
  float d1[4] = {0.f, 0.f, 0.f, 0.f}, d2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const float a0 = X[gid * ldx + 8 * ks + tig], a1 = X[(gid + 8) * ldx + 8 * ks + tig];
    const float a2 = X[gid * ldx + 8 * ks + tig + 4], a3 = X[(gid + 8) * ldx + 8 * ks + tig + 4];
    const float b0 = Y[(8 * ks + tig) * ldy + gid], b1 = Y[(8 * ks + tig + 4) * ldy + gid];
    const uint32_t ah[4] = {to_tf32(a0), to_tf32(a1), to_tf32(a2), to_tf32(a3)};
    const uint32_t al[4] = {to_tf32(a0 - __uint_as_float(ah[0])), to_tf32(a1 - __uint_as_float(ah[1])),
                            to_tf32(a2 - __uint_as_float(ah[2])), to_tf32(a3 - __uint_as_float(ah[3]))};
    const uint32_t bh[2] = {to_tf32(b0), to_tf32(b1)};
    const uint32_t bl[2] = {to_tf32(b0 - __uint_as_float(bh[0])), to_tf32(b1 - __uint_as_float(bh[1]))};
    mma_tf32_16x8x8(d, ah, bh);
    mma_tf32_16x8x8(d1, ah, bl);
    mma_tf32_16x8x8(d2, al, bh);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) d[e] += d1[e] + d2[e];
}
__device__ __forceinline__ void st_frag16x8(float *M, int ld, const float *d, float scale, int lane) {
  const int gid = lane >> 2, tig = lane & 3;
  M[gid * ld + 2 * tig] = scale * d[0];
  M[gid * ld + 2 * tig + 1] = scale * d[1];
  M[(gid + 8) * ld + 2 * tig] = scale * d[2];
  M[(gid + 8) * ld + 2 * tig + 1] = scale * d[3];
}

// Off-diagonal 16x16 blocks at block distance DIST (1..3) of the inverse: for
// the 4 - DIST blocks (i, j = i - DIST), Y_ij = sum_{j<=k<i} A_ik Tm_kj (one
// 16 x 16 DIST x 16 product), then Tm_ij = -Tm_ii Y_ij (16 x 16 x 16).  One warp
// per (block, 8-column half): the second product reads only the 8 columns of
// Y_ij the same warp wrote, so a warp barrier separates the two; NT threads
// (>= 192) meet at named barrier BAR once the distance is done.
template <int DIST, int NT, int BAR>
__device__ __forceinline__ void ut_distance(const float *__restrict__ A, float *__restrict__ Tm,
                                            float *__restrict__ Y, int etid) {
  constexpr int NB = 4 - DIST;
  const int w = etid >> 5, lane = etid & 31;
  if (w < 2 * NB) {
    const int j = w >> 1, i = j + DIST, nh = w & 1;
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    mma3_16x8<2 * DIST>(d, A + 16 * i * AST + 16 * j, AST, Tm + 16 * j * AST + 16 * j + 8 * nh, AST, lane);
    st_frag16x8(Y + (j * 16) * 17 + 8 * nh, 17, d, 1.f, lane);
    __syncwarp();
    float e[4] = {0.f, 0.f, 0.f, 0.f};
    mma3_16x8<2>(e, Tm + 16 * i * AST + 16 * i, AST, Y + (j * 16) * 17 + 8 * nh, 17, lane);
    st_frag16x8(Tm + 16 * i * AST + 16 * j + 8 * nh, AST, e, -1.f, lane);
  }
  named_bar_sync(BAR, NT);
}

// Unit lower-triangular inverse Tm = (I + A)^-1 of a 64x64 strictly lower A
// (fp32, shared memory, row stride AST), by NT = 256 or 512 threads.  The four
// 16x16 diagonal blocks by forward substitution: column c of block b is solved
// by one group of lanes that hold its rows (NT = 512: 8 lanes x 2 rows; NT =
// 256: 4 lanes x 4 rows; A read from shared memory), the solved entry of
// step s passed by a shuffle.  Then the off-diagonal blocks by
// block distance 1, 2, 3 (each needs only blocks of smaller distance), one
// block-wide barrier per distance.  Only
// the lower triangle of Tm is written.  Y holds [3][16][17] fp32 of scratch.
template <int NT, int BAR>
__device__ __forceinline__ void ut_solve(const float *__restrict__ A, float *__restrict__ Tm,
                                         float *__restrict__ Y, int etid) {
  static_assert(NT == 256 || NT == 512, "solve layouts exist for 256 and 512 threads");
  constexpr int RPL = 1024 / NT;  // rows per lane: 2 or 4
  constexpr int LPC = 16 / RPL;   // lanes per column: 8 or 4
  {
    const int ew = etid >> 5, lane = etid & 31;
    const int b = ew / (NT / 128);                                  // diagonal block
    const int c = (32 / LPC) * (ew % (NT / 128)) + lane / LPC;      // column within the block
    const int q = lane % LPC;                                       // rows q + LPC m
    const float *Ab = A + 16 * b * AST + 16 * b;
    float x[RPL];
#pragma unroll
    for (int m = 0; m < RPL; ++m) x[m] = (q + LPC * m == c) ? 1.f : 0.f;
#pragma unroll
    for (int s = 0; s < 16; ++s) {
      const float xs = __shfl_sync(0xffffffffu, x[s / LPC], (lane & ~(LPC - 1)) | (s % LPC));
#pragma unroll
      for (int m = 0; m < RPL; ++m) {
        const int r = q + LPC * m;
        if (r > s) x[m] = fmaf(-Ab[r * AST + s], xs, x[m]);
      }
    }
#pragma unroll
    for (int m = 0; m < RPL; ++m) Tm[(16 * b + q + LPC * m) * AST + 16 * b + c] = x[m];
  }
  named_bar_sync(BAR, NT);
  ut_distance<1, NT, BAR>(A, Tm, Y, etid);
  ut_distance<2, NT, BAR>(A, Tm, Y, etid);
  ut_distance<3, NT, BAR>(A, Tm, Y, etid);
}

// 8 consecutive fp32 values -> one 16-byte chunk of bf16 (round to nearest).
__device__ __forceinline__ uint4 pack_bf16x8(const float *x) {
  return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                    pack_bf16x2(x[6], x[7]));
}
__device__ __forceinline__ void st_bf16x8(unsigned char *dst, const float *x) {
  *reinterpret_cast<uint4 *>(dst) = pack_bf16x8(x);
}

// 2 NP fp32 values x -> packed bf16 pairs hw[NP] = hi(x), lw[NP] = lo(x):
// hi = x truncated to bf16 (its high 16 bits), lo = (x - hi) truncated to
// bf16; |x - hi - lo| < 2^-14 |x|.  Bit operations only (mask, subtract, byte
// permute), no conversion instructions.
template <int NP>
__device__ __forceinline__ void split_words(const float *x, uint32_t *hw, uint32_t *lw) {
#pragma unroll
  for (int e = 0; e < NP; ++e) {
    const uint32_t a = __float_as_uint(x[2 * e]), b = __float_as_uint(x[2 * e + 1]);
    const float ra = x[2 * e] - __uint_as_float(a & 0xffff0000u);
    const float rb = x[2 * e + 1] - __uint_as_float(b & 0xffff0000u);
    hw[e] = __byte_perm(a, b, 0x7632);
    lw[e] = __byte_perm(__float_as_uint(ra), __float_as_uint(rb), 0x7632);
  }
}
// The two halves of split_words separately: hi(x) words, then lo(x) words.
template <int NP>
__device__ __forceinline__ void hi_words(const float *x, uint32_t *hw) {
#pragma unroll
  for (int e = 0; e < NP; ++e)
    hw[e] = __byte_perm(__float_as_uint(x[2 * e]), __float_as_uint(x[2 * e + 1]), 0x7632);
}
template <int NP>
__device__ __forceinline__ void lo_words(const float *x, uint32_t *lw) {
#pragma unroll
  for (int e = 0; e < NP; ++e) {
    const float ra = x[2 * e] - __uint_as_float(__float_as_uint(x[2 * e]) & 0xffff0000u);
    const float rb = x[2 * e + 1] - __uint_as_float(__float_as_uint(x[2 * e + 1]) & 0xffff0000u);
    lw[e] = __byte_perm(__float_as_uint(ra), __float_as_uint(rb), 0x7632);
  }
}

// 8 fp32 values -> one 16-byte hi chunk and one 16-byte lo chunk.
__device__ __forceinline__ void st_split8(unsigned char *dst_hi, unsigned char *dst_lo,
                                          const float *x) {
  uint32_t hw[4], lw[4];
  split_words<4>(x, hw, lw);
  *reinterpret_cast<uint4 *>(dst_hi) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  *reinterpret_cast<uint4 *>(dst_lo) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
}

// Control words of a CTA in shared memory, as the tensor-core kernels lay
// them out: [0] the CTA's abort flag (any role may set it at any time), [1]
// the wait limit in microseconds, [2] the epilogue group's own abort word.
// The group acts only on [2], which nothing but the group's waiting thread
// writes, and only before the named barrier that publishes it: every thread
// of the group then reads the same value, so the group never splits across
// its named barriers (an abort seen only through [0] would let some threads
// leave while others wait at a barrier they never reach).
constexpr int CTL_ABORT = 0, CTL_LIMIT = 1, CTL_GROUP = 2;

// One waiter (thread 0 of the group) for an mbarrier phase, then a named
// barrier of the NT group threads; returns false once the group has given up,
// and then for every thread of the group.  (A waiter that gave up outside
// this helper sets both abort words: the group then stops here at the latest,
// whether or not this phase completed.)
template <int NT, int BAR>
__device__ __forceinline__ bool group_wait(uint32_t bar, uint32_t parity, int gtid,
                                           volatile int *ctl, int32_t *status) {
  if (gtid == 0 && !mbar_wait(bar, parity, ctl)) {
    ctl[CTL_ABORT] = 1;
    ctl[CTL_GROUP] = 1;
    report_status(status, GDN_ERR_DEVICE_TIMEOUT);
  }
  named_bar_sync(BAR, NT);
  const bool ok = ctl[CTL_GROUP] == 0;
  if (ok) tc_fence_after();
  return ok;
}

}  // namespace chunk
}  // namespace gdn
