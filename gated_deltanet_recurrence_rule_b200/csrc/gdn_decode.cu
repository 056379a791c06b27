// gdn_decode.cu -- one decode step of the gated delta rule for a batch of
// sequences, state updated in place.
//
// Per (sequence b, value head h), with S the Dv x Dk fp32 state, k and q of
// query/key head h / (Hv / Hqk), alpha = exp(g), beta the write strength:
//   u_i = S_i . k,  p_i = S_i . q          (both from the same pass over row i)
//   c_i = beta (v_i - alpha u_i)
//   S'_i = alpha S_i + c_i k^T             (= alpha S (I - beta k k^T) + beta v k^T, row i)
//   o_i  = scale (alpha p_i + c_i (k . q)) (= scale S' q)
// Token-by-token form of the rule described in "Inside Qwen3.8-27B: Hybrid
// DeltaNet Architecture, 256k Context, and 24GB Local Serving", section "Gated
// DeltaNet Mechanics" (inference updates the state one token at a time).
//
// The step is bound by HBM: each 64 KiB state is read once and written once
// (8 bytes per element against 3 FMAs).  Layout of the work:
//   - one 128-thread CTA per (b, h); warp w owns rows [w*Dv/4, (w+1)*Dv/4);
//   - 8 lanes cover one row, lane c8 holding the float4 chunks at columns
//     32 m + 4 c8 (m = 0 .. Dk/32-1), so one load instruction of a warp
//     reads four full 128-byte row segments;
//   - each lane keeps 4 row groups (16 float4) in flight before reducing;
//   - both dot products are reduced over the 8 lanes with 3 xor-shuffles
//     each, and the updated rows are written back with streaming stores.
#include "gdn_common.cuh"

namespace gdn {

template <typename T, typename TO, int DK, int DV>
__global__ void __launch_bounds__(128, 4)
decode_step_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                   const float *__restrict__ g, const float *__restrict__ beta,
                   float *__restrict__ state, TO *__restrict__ o, int Hqk, int Hv, float scale) {
  constexpr int NV4 = DK / 32;              // float4 chunks per lane per row
  constexpr int ROWS_PER_WARP = DV / 4;
  constexpr int GROUPS = ROWS_PER_WARP / 4;  // 4 rows per warp instruction
  constexpr int BATCH = GROUPS < 4 ? GROUPS : 4;
  static_assert(GROUPS % BATCH == 0, "row groups must split into batches");

  const int bh = blockIdx.x;
  const int b = bh / Hv, h = bh - b * Hv;
  const int j = h / (Hv / Hqk);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c8 = lane & 7, rr = lane >> 3;

  float kf[NV4 * 4], qf[NV4 * 4];
  const T *kp = k + ((size_t)b * Hqk + j) * DK;
  const T *qp = q + ((size_t)b * Hqk + j) * DK;
#pragma unroll
  for (int m = 0; m < NV4; ++m) {
    load4(kp + 32 * m + 4 * c8, kf + 4 * m);
    load4(qp + 32 * m + 4 * c8, qf + 4 * m);
  }
  float kap = 0.f;
#pragma unroll
  for (int x = 0; x < NV4 * 4; ++x) kap = fmaf(kf[x], qf[x], kap);
  kap += __shfl_xor_sync(0xffffffffu, kap, 1);
  kap += __shfl_xor_sync(0xffffffffu, kap, 2);
  kap += __shfl_xor_sync(0xffffffffu, kap, 4);

  const float alpha = expf(g[bh]);
  const float bt = beta[bh];
  const size_t row0 = (size_t)bh * DV + warp * ROWS_PER_WARP;
  float *S = state + row0 * DK;
  const float vreg = lane < ROWS_PER_WARP ? to_f32(v[row0 + lane]) : 0.f;
  float oreg = 0.f;

#pragma unroll
  for (int gb = 0; gb < GROUPS; gb += BATCH) {
    float4 s[BATCH][NV4];
#pragma unroll
    for (int x = 0; x < BATCH; ++x)
#pragma unroll
      for (int m = 0; m < NV4; ++m)
        s[x][m] = ld_stream(reinterpret_cast<const float4 *>(
            S + (size_t)((gb + x) * 4 + rr) * DK + 32 * m + 4 * c8));
#pragma unroll
    for (int x = 0; x < BATCH; ++x) {
      float u = 0.f, p = 0.f;
#pragma unroll
      for (int m = 0; m < NV4; ++m) {
        u = fmaf(s[x][m].x, kf[4 * m + 0], u); p = fmaf(s[x][m].x, qf[4 * m + 0], p);
        u = fmaf(s[x][m].y, kf[4 * m + 1], u); p = fmaf(s[x][m].y, qf[4 * m + 1], p);
        u = fmaf(s[x][m].z, kf[4 * m + 2], u); p = fmaf(s[x][m].z, qf[4 * m + 2], p);
        u = fmaf(s[x][m].w, kf[4 * m + 3], u); p = fmaf(s[x][m].w, qf[4 * m + 3], p);
      }
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) {
        u += __shfl_xor_sync(0xffffffffu, u, off);
        p += __shfl_xor_sync(0xffffffffu, p, off);
      }
      const int row = (gb + x) * 4 + rr;
      const float vi = __shfl_sync(0xffffffffu, vreg, row);
      const float c = bt * (vi - alpha * u);
      const float oi = fmaf(alpha, p, c * kap);
#pragma unroll
      for (int m = 0; m < NV4; ++m) {
        float4 y;
        y.x = fmaf(alpha, s[x][m].x, c * kf[4 * m + 0]);
        y.y = fmaf(alpha, s[x][m].y, c * kf[4 * m + 1]);
        y.z = fmaf(alpha, s[x][m].z, c * kf[4 * m + 2]);
        y.w = fmaf(alpha, s[x][m].w, c * kf[4 * m + 3]);
        st_stream(reinterpret_cast<float4 *>(S + (size_t)row * DK + 32 * m + 4 * c8), y);
      }
      // lane L collects the output of row L (row group L/4, row L%4 in it)
      const float og = __shfl_sync(0xffffffffu, oi, (lane & 3) * 8);
      if ((lane >> 2) == gb + x) oreg = og;
    }
  }
  if (lane < ROWS_PER_WARP) o[row0 + lane] = from_f32<TO>(scale * oreg);
}

template <typename T, typename TO, int DK, int DV>
static cudaError_t launch_decode_t(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, float *state, void *o, int B, int Hqk,
                                   int Hv, float scale, cudaStream_t stream) {
  const unsigned blocks = (unsigned)B * (unsigned)Hv;
  decode_step_kernel<T, TO, DK, DV><<<blocks, 128, 0, stream>>>(
      static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), g, beta,
      state, static_cast<TO *>(o), Hqk, Hv, scale);
  return cudaGetLastError();
}

cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float *state, void *o, int B, int Hqk, int Hv,
                          int Dk, int Dv, int dtype, int o_dtype, float scale,
                          cudaStream_t s) {
  return dispatch_types(dtype, o_dtype, [&](auto t, auto to) {
    using T = decltype(t);
    using TO = decltype(to);
    if (Dk == 128 && Dv == 128) return launch_decode_t<T, TO, 128, 128>(q, k, v, g, beta, state, o, B, Hqk, Hv, scale, s);
    if (Dk == 128 && Dv == 64) return launch_decode_t<T, TO, 128, 64>(q, k, v, g, beta, state, o, B, Hqk, Hv, scale, s);
    if (Dk == 64 && Dv == 128) return launch_decode_t<T, TO, 64, 128>(q, k, v, g, beta, state, o, B, Hqk, Hv, scale, s);
    return launch_decode_t<T, TO, 64, 64>(q, k, v, g, beta, state, o, B, Hqk, Hv, scale, s);
  });
}


// ---------------------------------------------------------------------------
// Several tokens per sequence in one call, states in a slot pool.
//
// For each sequence b and value head h: S <- state_in[src_slot[b], h]; then for
// t = 0 .. Tn-1 the same token step as above; finally state_out[dst_slot[b], h]
// <- S.  Every state row is updated Tn times in registers between one read and
// one write, so the HBM bytes per call stay those of one step while the tokens
// grow Tn-fold (multi-token decode, e.g. verifying a few speculated tokens).
// The per-token k and q (fp32) are staged in shared memory; each lane reads its
// 16 columns of them per token.  Outputs are stored by the first lane of each
// row's 8-lane group.
namespace {
constexpr int kMaxTokens = 16;
}

template <typename T, typename TO, int DK, int DV>
__global__ void __launch_bounds__(128, 4)
decode_tokens_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                     const float *__restrict__ g, const float *__restrict__ beta,
                     const float *state_in, float *state_out, const int32_t *__restrict__ src_slot,
                     const int32_t *__restrict__ dst_slot, int num_slots, TO *__restrict__ o,
                     int Tn, int Hqk, int Hv, float scale, int32_t *status) {
  constexpr int NV4 = DK / 32;
  constexpr int ROWS_PER_WARP = DV / 4;
  constexpr int GROUPS = ROWS_PER_WARP / 4;
  constexpr int BATCH = GROUPS < 4 ? GROUPS : 4;
  static_assert(GROUPS % BATCH == 0, "row groups must split into batches");
  __shared__ __align__(16) float kq[kMaxTokens][2][DK];  // k_t, q_t
  __shared__ float tok[kMaxTokens][2];                    // alpha_t, beta_t

  const int b = blockIdx.x / Hv, h = blockIdx.x - (blockIdx.x / Hv) * Hv;
  const int j = h / (Hv / Hqk);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c8 = lane & 7, rr = lane >> 3;
  const int src = src_slot ? src_slot[b] : b;
  const int dst = dst_slot ? dst_slot[b] : src;
  if (src < 0) return;  // padding entry: nothing read or written
  if (src >= num_slots || dst < 0 || dst >= num_slots) {
    if (threadIdx.x == 0) report_status(status, GDN_ERR_INVALID_ARG);
    return;
  }

  // stage k_t, q_t (fp32) and the per-token scalars
  for (int x = threadIdx.x; x < Tn * DK; x += blockDim.x) {
    const int t = x / DK, d = x - t * DK;
    const size_t off = (((size_t)b * Tn + t) * Hqk + j) * DK + d;
    kq[t][0][d] = to_f32(k[off]);
    kq[t][1][d] = to_f32(q[off]);
  }
  __syncthreads();
  for (int t = threadIdx.x; t < Tn; t += blockDim.x) {
    const size_t gi = ((size_t)b * Tn + t) * Hv + h;
    tok[t][0] = expf(g[gi]);
    tok[t][1] = beta[gi];
  }
  __syncthreads();

  const size_t rowS = (size_t)h * DV + warp * ROWS_PER_WARP;  // first row of this warp in a slot
  const float *Sin = state_in + ((size_t)src * Hv * DV + rowS) * DK;
  float *Sout = state_out + ((size_t)dst * Hv * DV + rowS) * DK;

#pragma unroll
  for (int gb = 0; gb < GROUPS; gb += BATCH) {
    float4 s[BATCH][NV4];
#pragma unroll
    for (int x = 0; x < BATCH; ++x)
#pragma unroll
      for (int m = 0; m < NV4; ++m)
        s[x][m] = ld_stream(reinterpret_cast<const float4 *>(
            Sin + (size_t)((gb + x) * 4 + rr) * DK + 32 * m + 4 * c8));
    for (int t = 0; t < Tn; ++t) {
      float kf[NV4 * 4], qf[NV4 * 4];
#pragma unroll
      for (int m = 0; m < NV4; ++m) {
        const float4 a = *reinterpret_cast<const float4 *>(&kq[t][0][32 * m + 4 * c8]);
        const float4 c = *reinterpret_cast<const float4 *>(&kq[t][1][32 * m + 4 * c8]);
        kf[4 * m] = a.x; kf[4 * m + 1] = a.y; kf[4 * m + 2] = a.z; kf[4 * m + 3] = a.w;
        qf[4 * m] = c.x; qf[4 * m + 1] = c.y; qf[4 * m + 2] = c.z; qf[4 * m + 3] = c.w;
      }
      // k . q as the single-token step forms it: lane partials, 8-lane reduction
      float kap = 0.f;
#pragma unroll
      for (int x = 0; x < NV4 * 4; ++x) kap = fmaf(kf[x], qf[x], kap);
      kap += __shfl_xor_sync(0xffffffffu, kap, 1);
      kap += __shfl_xor_sync(0xffffffffu, kap, 2);
      kap += __shfl_xor_sync(0xffffffffu, kap, 4);
      const float alpha = tok[t][0], bt = tok[t][1];
      const size_t vrow = (((size_t)b * Tn + t) * Hv + h) * DV + warp * ROWS_PER_WARP;
#pragma unroll
      for (int x = 0; x < BATCH; ++x) {
        float u = 0.f, p = 0.f;
#pragma unroll
        for (int m = 0; m < NV4; ++m) {
          u = fmaf(s[x][m].x, kf[4 * m + 0], u); p = fmaf(s[x][m].x, qf[4 * m + 0], p);
          u = fmaf(s[x][m].y, kf[4 * m + 1], u); p = fmaf(s[x][m].y, qf[4 * m + 1], p);
          u = fmaf(s[x][m].z, kf[4 * m + 2], u); p = fmaf(s[x][m].z, qf[4 * m + 2], p);
          u = fmaf(s[x][m].w, kf[4 * m + 3], u); p = fmaf(s[x][m].w, qf[4 * m + 3], p);
        }
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) {
          u += __shfl_xor_sync(0xffffffffu, u, off);
          p += __shfl_xor_sync(0xffffffffu, p, off);
        }
        const int row = (gb + x) * 4 + rr;
        const float vi = to_f32(v[vrow + row]);
        const float c = bt * (vi - alpha * u);
        if (c8 == 0) o[vrow + row] = from_f32<TO>(scale * fmaf(alpha, p, c * kap));
#pragma unroll
        for (int m = 0; m < NV4; ++m) {
          s[x][m].x = fmaf(alpha, s[x][m].x, c * kf[4 * m + 0]);
          s[x][m].y = fmaf(alpha, s[x][m].y, c * kf[4 * m + 1]);
          s[x][m].z = fmaf(alpha, s[x][m].z, c * kf[4 * m + 2]);
          s[x][m].w = fmaf(alpha, s[x][m].w, c * kf[4 * m + 3]);
        }
      }
    }
#pragma unroll
    for (int x = 0; x < BATCH; ++x)
#pragma unroll
      for (int m = 0; m < NV4; ++m)
        st_stream(reinterpret_cast<float4 *>(Sout + (size_t)((gb + x) * 4 + rr) * DK + 32 * m + 4 * c8),
                  s[x][m]);
  }
}

template <typename T, typename TO, int DK, int DV>
static cudaError_t launch_decode_tokens_t(const void *q, const void *k, const void *v,
                                          const float *g, const float *beta, const float *sin,
                                          float *sout, const int32_t *src, const int32_t *dst,
                                          int num_slots, void *o, int B, int Tn, int Hqk, int Hv,
                                          float scale, int32_t *status, cudaStream_t stream) {
  const unsigned blocks = (unsigned)B * (unsigned)Hv;
  decode_tokens_kernel<T, TO, DK, DV><<<blocks, 128, 0, stream>>>(
      static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), g, beta, sin,
      sout, src, dst, num_slots, static_cast<TO *>(o), Tn, Hqk, Hv, scale, status);
  return cudaGetLastError();
}

int decode_tokens_max() { return kMaxTokens; }

cudaError_t launch_decode_tokens(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *state_in, float *state_out,
                                 const int32_t *src_slot, const int32_t *dst_slot, int num_slots,
                                 void *o, int B, int Tn, int Hqk, int Hv, int Dk, int Dv, int dtype,
                                 int o_dtype, float scale, int32_t *status, cudaStream_t s) {
  return dispatch_types(dtype, o_dtype, [&](auto t, auto to) {
    using T = decltype(t);
    using TO = decltype(to);
    if (Dk == 128 && Dv == 128)
      return launch_decode_tokens_t<T, TO, 128, 128>(q, k, v, g, beta, state_in, state_out, src_slot, dst_slot, num_slots, o, B, Tn, Hqk, Hv, scale, status, s);
    if (Dk == 128 && Dv == 64)
      return launch_decode_tokens_t<T, TO, 128, 64>(q, k, v, g, beta, state_in, state_out, src_slot, dst_slot, num_slots, o, B, Tn, Hqk, Hv, scale, status, s);
    if (Dk == 64 && Dv == 128)
      return launch_decode_tokens_t<T, TO, 64, 128>(q, k, v, g, beta, state_in, state_out, src_slot, dst_slot, num_slots, o, B, Tn, Hqk, Hv, scale, status, s);
    return launch_decode_tokens_t<T, TO, 64, 64>(q, k, v, g, beta, state_in, state_out, src_slot, dst_slot, num_slots, o, B, Tn, Hqk, Hv, scale, status, s);
  });
}

}  // namespace gdn
