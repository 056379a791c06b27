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
  pdl_wait();  // nothing is read before the previous kernel on the stream is done
  pdl_allow_next();
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
  return launch_pdl(decode_step_kernel<T, TO, DK, DV>, blocks, 128, 0, stream,
                    static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v),
                    g, beta, state, static_cast<TO *>(o), Hqk, Hv, scale);
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
// The per-token k, q and v (fp32) are staged in shared memory, so that no
// global load sits in the dependent chain of a token update; each lane reads
// its 16 columns of k and q per token.  Outputs are stored by the first lane of
// each row's 8-lane group.
namespace {
constexpr int kMaxTokens = 16;
}

template <typename T, typename TO, int DK, int DV>
__global__ void __launch_bounds__(128, 4)
decode_tokens_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                     const float *__restrict__ g, const float *__restrict__ beta,
                     const float *state_in, float *state_out, const int32_t *__restrict__ src_slot,
                     const int32_t *__restrict__ dst_slot, int num_slots, TO *__restrict__ o,
                     int Tn, int Hqk, int Hv, float scale, int32_t *status, int raw) {
  pdl_wait();  // nothing is read before the previous kernel on the stream is done
  pdl_allow_next();
  constexpr int NV4 = DK / 32;
  constexpr int ROWS_PER_WARP = DV / 4;
  constexpr int GROUPS = ROWS_PER_WARP / 4;
  constexpr int BATCH = GROUPS < 4 ? GROUPS : 4;
  static_assert(GROUPS % BATCH == 0, "row groups must split into batches");
  __shared__ __align__(16) float kq[kMaxTokens][2][DK];  // k_t, q_t
  __shared__ float vs[kMaxTokens][DV];                    // v_t of this value head
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

  const size_t rowS = (size_t)h * DV + warp * ROWS_PER_WARP;  // first row of this warp in a slot
  const float *Sin = state_in + ((size_t)src * Hv * DV + rowS) * DK;
  float *Sout = state_out + ((size_t)dst * Hv * DV + rowS) * DK;
  float4 s[BATCH][NV4];
  auto load_batch = [&](int gb) {
#pragma unroll
    for (int x = 0; x < BATCH; ++x)
#pragma unroll
      for (int m = 0; m < NV4; ++m)
        s[x][m] = ld_stream(reinterpret_cast<const float4 *>(
            Sin + (size_t)((gb + x) * 4 + rr) * DK + 32 * m + 4 * c8));
  };
  load_batch(0);  // in flight while the tokens are staged

  // stage k_t, q_t, v_t (fp32) and the per-token scalars
  for (int x = threadIdx.x; x < Tn * DK; x += blockDim.x) {
    const int t = x / DK, d = x - t * DK;
    const size_t off = (((size_t)b * Tn + t) * Hqk + j) * DK + d;
    kq[t][0][d] = to_f32(k[off]);
    kq[t][1][d] = to_f32(q[off]);
  }
  for (int x = threadIdx.x; x < Tn * DV; x += blockDim.x) {
    const int t = x / DV, d = x - t * DV;
    vs[t][d] = to_f32(v[(((size_t)b * Tn + t) * Hv + h) * DV + d]);
  }
  for (int t = threadIdx.x; t < Tn; t += blockDim.x) {
    const size_t gi = ((size_t)b * Tn + t) * Hv + h;
    tok[t][0] = raw ? alpha_raw(g[gi]) : expf(g[gi]);
    tok[t][1] = raw ? beta_raw(beta[gi]) : beta[gi];
  }
  __syncthreads();
  if (raw) {  // unit L2 norm per token for k and q, one token per warp in turn
    for (int t = warp; t < Tn; t += 4) {
      float sk = 0.f, sq = 0.f;
      for (int d = lane; d < DK; d += 32) {
        sk = fmaf(kq[t][0][d], kq[t][0][d], sk);
        sq = fmaf(kq[t][1][d], kq[t][1][d], sq);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        sk += __shfl_xor_sync(0xffffffffu, sk, off);
        sq += __shfl_xor_sync(0xffffffffu, sq, off);
      }
      const float rk = inv_norm(sk), rq = inv_norm(sq);
      for (int d = lane; d < DK; d += 32) {
        kq[t][0][d] *= rk;
        kq[t][1][d] *= rq;
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int gb = 0; gb < GROUPS; gb += BATCH) {
    if (gb > 0) load_batch(gb);
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
        const float vi = vs[t][warp * ROWS_PER_WARP + row];
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

// The same multi-token step with the states at rest in bf16.  A state is read
// as bf16, widened to fp32 (exactly), updated for all of the call's tokens in
// fp32 registers, and rounded to bf16 (round to nearest even) once, when it is
// stored: a call of Tn tokens rounds each state once.  Per lane, 8 lanes per
// row, lane c8 holding the 16-byte pieces at columns 64 m + 8 c8 + (0..7), so
// one load instruction of a warp still covers four full 128-byte row segments.
// Each warp requests all of its rows (8 KiB at Dk = Dv = 128) before the tokens
// are staged, then updates them two row groups (8 rows) at a time, so that the
// k and q a lane reads from shared memory per token serve 8 rows.  k and q are
// staged in the lanes' column order (the float4 that lane c8 reads i-th sits at
// 32 i + 4 c8), so those reads are free of bank conflicts.
template <typename T, typename TO, int DK, int DV>
__global__ void __launch_bounds__(128, 3)
decode_tokens_bf16s_kernel(const T *__restrict__ q, const T *__restrict__ k,
                           const T *__restrict__ v, const float *__restrict__ g,
                           const float *__restrict__ beta, const __nv_bfloat16 *state_in,
                           __nv_bfloat16 *state_out, const int32_t *__restrict__ src_slot,
                           const int32_t *__restrict__ dst_slot, int num_slots,
                           TO *__restrict__ o, int Tn, int Hqk, int Hv, float scale,
                           int32_t *status, int raw) {
  pdl_wait();  // nothing is read before the previous kernel on the stream is done
  pdl_allow_next();
  constexpr int NU = DK / 64;  // 16-byte pieces per lane per row
  constexpr int E = NU * 8;    // state elements per lane per row
  constexpr int ROWS_PER_WARP = DV / 4;
  constexpr int GROUPS = ROWS_PER_WARP / 4;  // 4 rows per warp instruction
  constexpr int STAGE = 2;                   // row groups updated together
  static_assert(GROUPS % STAGE == 0, "row groups must split into stages");
  __shared__ __align__(16) float kq[kMaxTokens][2][DK];  // k_t, q_t in lane order
  __shared__ float vs[kMaxTokens][DV];                    // v_t of this value head
  __shared__ float tok[kMaxTokens][3];                    // alpha_t, beta_t, k_t . q_t

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

  const size_t rowS = (size_t)h * DV + warp * ROWS_PER_WARP;  // first row of this warp in a slot
  const __nv_bfloat16 *Sin = state_in + ((size_t)src * Hv * DV + rowS) * DK;
  __nv_bfloat16 *Sout = state_out + ((size_t)dst * Hv * DV + rowS) * DK;
  uint4 packed[GROUPS][NU];
#pragma unroll
  for (int x = 0; x < GROUPS; ++x)
#pragma unroll
    for (int m = 0; m < NU; ++m)
      packed[x][m] = __ldcs(reinterpret_cast<const uint4 *>(Sin + (size_t)(x * 4 + rr) * DK + 64 * m + 8 * c8));

  // stage k_t, q_t (fp32, column d = 64 m + 8 c + 4 hf + e at 32 (2 m + hf) + 4 c + e),
  // v_t and the per-token scalars
  for (int x = threadIdx.x; x < Tn * DK; x += blockDim.x) {
    const int t = x / DK, d = x - t * DK;
    const size_t off = (((size_t)b * Tn + t) * Hqk + j) * DK + d;
    const int pos = 32 * (2 * (d >> 6) + ((d >> 2) & 1)) + 4 * ((d >> 3) & 7) + (d & 3);
    kq[t][0][pos] = to_f32(k[off]);
    kq[t][1][pos] = to_f32(q[off]);
  }
  for (int x = threadIdx.x; x < Tn * DV; x += blockDim.x) {
    const int t = x / DV, d = x - t * DV;
    vs[t][d] = to_f32(v[(((size_t)b * Tn + t) * Hv + h) * DV + d]);
  }
  for (int t = threadIdx.x; t < Tn; t += blockDim.x) {
    const size_t gi = ((size_t)b * Tn + t) * Hv + h;
    tok[t][0] = raw ? alpha_raw(g[gi]) : expf(g[gi]);
    tok[t][1] = raw ? beta_raw(beta[gi]) : beta[gi];
  }
  __syncthreads();
  for (int t = warp; t < Tn; t += 4) {  // k_t . q_t, one token per warp in turn
    if (raw) {  // unit L2 norm for k_t and q_t first (order of columns is immaterial)
      float sk = 0.f, sq = 0.f;
      for (int d = lane; d < DK; d += 32) {
        sk = fmaf(kq[t][0][d], kq[t][0][d], sk);
        sq = fmaf(kq[t][1][d], kq[t][1][d], sq);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        sk += __shfl_xor_sync(0xffffffffu, sk, off);
        sq += __shfl_xor_sync(0xffffffffu, sq, off);
      }
      const float rk = inv_norm(sk), rq = inv_norm(sq);
      for (int d = lane; d < DK; d += 32) {
        kq[t][0][d] *= rk;
        kq[t][1][d] *= rq;
      }
    }
    float a = 0.f;
    for (int d = lane; d < DK; d += 32) a = fmaf(kq[t][0][d], kq[t][1][d], a);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
    if (lane == 0) tok[t][2] = a;
  }
  __syncthreads();

#pragma unroll
  for (int gs = 0; gs < GROUPS; gs += STAGE) {
    float2 s[STAGE][E / 2];  // adjacent columns in pairs, for the packed fp32x2 FMA
#pragma unroll
    for (int x = 0; x < STAGE; ++x)
#pragma unroll
      for (int m = 0; m < NU; ++m) {
        const uint32_t w[4] = {packed[gs + x][m].x, packed[gs + x][m].y, packed[gs + x][m].z,
                               packed[gs + x][m].w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          s[x][4 * m + i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
      }
    for (int t = 0; t < Tn; ++t) {
      float2 kf[E / 2], qf[E / 2];  // pair 2 i + (0, 1) of this lane's columns
#pragma unroll
      for (int i = 0; i < E / 4; ++i) {
        const float4 a = *reinterpret_cast<const float4 *>(&kq[t][0][32 * i + 4 * c8]);
        const float4 c = *reinterpret_cast<const float4 *>(&kq[t][1][32 * i + 4 * c8]);
        kf[2 * i] = make_float2(a.x, a.y); kf[2 * i + 1] = make_float2(a.z, a.w);
        qf[2 * i] = make_float2(c.x, c.y); qf[2 * i + 1] = make_float2(c.z, c.w);
      }
      const float alpha = tok[t][0], bt = tok[t][1], kap = tok[t][2];
      const float2 alpha2 = make_float2(alpha, alpha);
      const size_t orow = (((size_t)b * Tn + t) * Hv + h) * DV + warp * ROWS_PER_WARP;
#pragma unroll
      for (int x = 0; x < STAGE; ++x) {
        float2 u2 = make_float2(0.f, 0.f), p2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < E / 2; ++e) {
          u2 = __ffma2_rn(s[x][e], kf[e], u2);
          p2 = __ffma2_rn(s[x][e], qf[e], p2);
        }
        float u = u2.x + u2.y, p = p2.x + p2.y;
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) {
          u += __shfl_xor_sync(0xffffffffu, u, off);
          p += __shfl_xor_sync(0xffffffffu, p, off);
        }
        const int row = (gs + x) * 4 + rr;
        const float c = bt * (vs[t][warp * ROWS_PER_WARP + row] - alpha * u);
        if (c8 == 0) o[orow + row] = from_f32<TO>(scale * fmaf(alpha, p, c * kap));
        const float2 c2 = make_float2(c, c);
#pragma unroll
        for (int e = 0; e < E / 2; ++e) s[x][e] = __ffma2_rn(alpha2, s[x][e], __fmul2_rn(c2, kf[e]));
      }
    }
#pragma unroll
    for (int x = 0; x < STAGE; ++x)
#pragma unroll
      for (int m = 0; m < NU; ++m) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __nv_bfloat162 pr = __floats2bfloat162_rn(s[x][4 * m + i].x, s[x][4 * m + i].y);
          w[i] = *reinterpret_cast<const uint32_t *>(&pr);
        }
        __stcs(reinterpret_cast<uint4 *>(Sout + (size_t)((gs + x) * 4 + rr) * DK + 64 * m + 8 * c8),
               make_uint4(w[0], w[1], w[2], w[3]));
      }
  }
}

// One token per sequence against a bf16 pool (the decode step with states at
// rest in bf16).  Same arithmetic as the kernel above at Tn = 1, laid out like
// the fp32 decode step: k, q and v go straight from global memory into
// registers (no shared memory, no block barrier) and every warp has all of its
// rows in flight (8 KiB at Dk = Dv = 128) before the first one is used.
template <typename T, typename TO, int DK, int DV, bool RAW>
__global__ void __launch_bounds__(128, RAW ? 3 : 4)  // the prologue needs a few more registers
decode_one_bf16s_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                        const float *__restrict__ g, const float *__restrict__ beta,
                        const __nv_bfloat16 *state_in, __nv_bfloat16 *state_out,
                        const int32_t *__restrict__ src_slot, const int32_t *__restrict__ dst_slot,
                        int num_slots, TO *__restrict__ o, int Hqk, int Hv, float scale,
                        int32_t *status) {
  pdl_wait();  // nothing is read before the previous kernel on the stream is done
  pdl_allow_next();
  constexpr int NU = DK / 64;  // 16-byte pieces per lane per row
  constexpr int E = NU * 8;    // state elements per lane per row
  constexpr int ROWS_PER_WARP = DV / 4;
  constexpr int GROUPS = ROWS_PER_WARP / 4;  // 4 rows per warp instruction

  const int bh = blockIdx.x;
  const int b = bh / Hv, h = bh - b * Hv;
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

  const size_t rowS = (size_t)h * DV + warp * ROWS_PER_WARP;  // first row of this warp in a slot
  const __nv_bfloat16 *Sin = state_in + ((size_t)src * Hv * DV + rowS) * DK;
  __nv_bfloat16 *Sout = state_out + ((size_t)dst * Hv * DV + rowS) * DK;
  uint4 packed[GROUPS][NU];
#pragma unroll
  for (int x = 0; x < GROUPS; ++x)
#pragma unroll
    for (int m = 0; m < NU; ++m)
      packed[x][m] = __ldcs(reinterpret_cast<const uint4 *>(Sin + (size_t)(x * 4 + rr) * DK + 64 * m + 8 * c8));

  float2 kf[E / 2], qf[E / 2];  // columns 64 m + 8 c8 + (0..7), in pairs
  const T *kp = k + ((size_t)b * Hqk + j) * DK;
  const T *qp = q + ((size_t)b * Hqk + j) * DK;
#pragma unroll
  for (int m = 0; m < NU; ++m)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float a[4], c[4];
      load4(kp + 64 * m + 8 * c8 + 4 * hf, a);
      load4(qp + 64 * m + 8 * c8 + 4 * hf, c);
      kf[4 * m + 2 * hf] = make_float2(a[0], a[1]); kf[4 * m + 2 * hf + 1] = make_float2(a[2], a[3]);
      qf[4 * m + 2 * hf] = make_float2(c[0], c[1]); qf[4 * m + 2 * hf + 1] = make_float2(c[2], c[3]);
    }
  if constexpr (RAW) {  // unit L2 norm: the 8 lanes of a row group hold all Dk columns
    float2 sk2 = make_float2(0.f, 0.f), sq2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int e = 0; e < E / 2; ++e) {
      sk2 = __ffma2_rn(kf[e], kf[e], sk2);
      sq2 = __ffma2_rn(qf[e], qf[e], sq2);
    }
    float sk = sk2.x + sk2.y, sq = sq2.x + sq2.y;
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
      sk += __shfl_xor_sync(0xffffffffu, sk, off);
      sq += __shfl_xor_sync(0xffffffffu, sq, off);
    }
    const float2 rk = make_float2(inv_norm(sk), inv_norm(sk)), rq = make_float2(inv_norm(sq), inv_norm(sq));
#pragma unroll
    for (int e = 0; e < E / 2; ++e) {
      kf[e] = __fmul2_rn(kf[e], rk);
      qf[e] = __fmul2_rn(qf[e], rq);
    }
  }
  float2 kap2 = make_float2(0.f, 0.f);
#pragma unroll
  for (int e = 0; e < E / 2; ++e) kap2 = __ffma2_rn(kf[e], qf[e], kap2);
  float kap = kap2.x + kap2.y;
  kap += __shfl_xor_sync(0xffffffffu, kap, 1);
  kap += __shfl_xor_sync(0xffffffffu, kap, 2);
  kap += __shfl_xor_sync(0xffffffffu, kap, 4);

  const float alpha = RAW ? alpha_raw(g[bh]) : expf(g[bh]);
  const float bt = RAW ? beta_raw(beta[bh]) : beta[bh];
  const float2 alpha2 = make_float2(alpha, alpha);
  const size_t row0 = (size_t)bh * DV + warp * ROWS_PER_WARP;  // o and v rows of this warp
  const float vreg = lane < ROWS_PER_WARP ? to_f32(v[row0 + lane]) : 0.f;
  float oreg = 0.f;

#pragma unroll
  for (int x = 0; x < GROUPS; ++x) {
    float2 s[E / 2];
#pragma unroll
    for (int m = 0; m < NU; ++m) {
      const uint32_t w[4] = {packed[x][m].x, packed[x][m].y, packed[x][m].z, packed[x][m].w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        s[4 * m + i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
    }
    float2 u2 = make_float2(0.f, 0.f), p2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int e = 0; e < E / 2; ++e) {
      u2 = __ffma2_rn(s[e], kf[e], u2);
      p2 = __ffma2_rn(s[e], qf[e], p2);
    }
    float u = u2.x + u2.y, p = p2.x + p2.y;
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
      u += __shfl_xor_sync(0xffffffffu, u, off);
      p += __shfl_xor_sync(0xffffffffu, p, off);
    }
    const int row = x * 4 + rr;
    const float vi = __shfl_sync(0xffffffffu, vreg, row);
    const float c = bt * (vi - alpha * u);
    const float oi = fmaf(alpha, p, c * kap);
    const float2 c2 = make_float2(c, c);
#pragma unroll
    for (int m = 0; m < NU; ++m) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 y = __ffma2_rn(alpha2, s[4 * m + i], __fmul2_rn(c2, kf[4 * m + i]));
        const __nv_bfloat162 pr = __floats2bfloat162_rn(y.x, y.y);
        w[i] = *reinterpret_cast<const uint32_t *>(&pr);
      }
      __stcs(reinterpret_cast<uint4 *>(Sout + (size_t)row * DK + 64 * m + 8 * c8),
             make_uint4(w[0], w[1], w[2], w[3]));
    }
    // lane L collects the output of row L (row group L/4, row L%4 in it)
    const float og = __shfl_sync(0xffffffffu, oi, (lane & 3) * 8);
    if ((lane >> 2) == x) oreg = og;
  }
  if (lane < ROWS_PER_WARP) o[row0 + lane] = from_f32<TO>(scale * oreg);
}

template <typename T, typename TO, int DK, int DV>
static cudaError_t launch_decode_tokens_t(const void *q, const void *k, const void *v,
                                          const float *g, const float *beta, const void *sin,
                                          void *sout, const int32_t *src, const int32_t *dst,
                                          int num_slots, void *o, int B, int Tn, int Hqk, int Hv,
                                          float scale, int state_dtype, int raw, int32_t *status,
                                          cudaStream_t stream) {
  const unsigned blocks = (unsigned)B * (unsigned)Hv;
  const T *qt = static_cast<const T *>(q), *kt = static_cast<const T *>(k),
          *vt = static_cast<const T *>(v);
  TO *ot = static_cast<TO *>(o);
  if (state_dtype == GDN_DTYPE_BF16 && Tn == 1)  // the input form is compiled in: registers are tight
    return launch_pdl(raw ? decode_one_bf16s_kernel<T, TO, DK, DV, true>
                          : decode_one_bf16s_kernel<T, TO, DK, DV, false>,
                      blocks, 128, 0, stream, qt, kt, vt, g, beta,
                      static_cast<const __nv_bfloat16 *>(sin), static_cast<__nv_bfloat16 *>(sout),
                      src, dst, num_slots, ot, Hqk, Hv, scale, status);
  if (state_dtype == GDN_DTYPE_BF16)
    return launch_pdl(decode_tokens_bf16s_kernel<T, TO, DK, DV>, blocks, 128, 0, stream, qt, kt,
                      vt, g, beta, static_cast<const __nv_bfloat16 *>(sin),
                      static_cast<__nv_bfloat16 *>(sout), src, dst, num_slots, ot, Tn, Hqk, Hv,
                      scale, status, raw);
  return launch_pdl(decode_tokens_kernel<T, TO, DK, DV>, blocks, 128, 0, stream, qt, kt, vt, g,
                    beta, static_cast<const float *>(sin), static_cast<float *>(sout), src, dst,
                    num_slots, ot, Tn, Hqk, Hv, scale, status, raw);
}

int decode_tokens_max() { return kMaxTokens; }

cudaError_t launch_decode_tokens(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const void *state_in, void *state_out,
                                 const int32_t *src_slot, const int32_t *dst_slot, int num_slots,
                                 void *o, int B, int Tn, int Hqk, int Hv, int Dk, int Dv, int dtype,
                                 int o_dtype, int state_dtype, int input_form, float scale,
                                 int32_t *status, cudaStream_t s) {
  const int raw = input_form == GDN_INPUT_RAW;
  return dispatch_types(dtype, o_dtype, [&](auto t, auto to) {
    using T = decltype(t);
    using TO = decltype(to);
    if (Dk == 128 && Dv == 128)
      return launch_decode_tokens_t<T, TO, 128, 128>(q, k, v, g, beta, state_in, state_out, src_slot, dst_slot, num_slots, o, B, Tn, Hqk, Hv, scale, state_dtype, raw, status, s);
    if (Dk == 128 && Dv == 64)
      return launch_decode_tokens_t<T, TO, 128, 64>(q, k, v, g, beta, state_in, state_out, src_slot, dst_slot, num_slots, o, B, Tn, Hqk, Hv, scale, state_dtype, raw, status, s);
    if (Dk == 64 && Dv == 128)
      return launch_decode_tokens_t<T, TO, 64, 128>(q, k, v, g, beta, state_in, state_out, src_slot, dst_slot, num_slots, o, B, Tn, Hqk, Hv, scale, state_dtype, raw, status, s);
    return launch_decode_tokens_t<T, TO, 64, 64>(q, k, v, g, beta, state_in, state_out, src_slot, dst_slot, num_slots, o, B, Tn, Hqk, Hv, scale, state_dtype, raw, status, s);
  });
}

}  // namespace gdn
