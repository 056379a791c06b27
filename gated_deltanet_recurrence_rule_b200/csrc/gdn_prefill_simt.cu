// gdn_prefill_simt.cu -- fp32 CUDA-core prefill of the gated delta rule.
//
// The token-by-token recurrence ("Inside Qwen3.8-27B: Hybrid DeltaNet
// Architecture, 256k Context, and 24GB Local Serving", section "Gated DeltaNet
// Mechanics"), computed in fp32 with the state in registers:
//   u_i = S_i . k_t;  S_i <- alpha_t S_i + beta_t (v_ti - alpha_t u_i) k_t^T;  o_ti = scale S_i . q_t
// This kernel serves fp32 inputs (whose tolerance, 1e-4 relative, tensor-core
// tf32 cannot meet), head dims other than 128, and any call the tensor-core
// kernel does not take.
//
// Work split: one 128-thread CTA per (sequence, value head, 32-row slice of
// the state).  Rows of S evolve independently given k, so slices need no
// communication.  Four lanes share a row, each holding Dk/4 columns as
// float4 chunks at columns 16 m + 4 r (r = lane & 3), which keeps the
// shared-memory reads of k and q conflict-free.  Inputs for 16 tokens at a
// time are copied to shared memory with cp.async (double buffered), then
// converted to fp32 once per stage.
#include "gdn_common.cuh"

namespace gdn {

namespace {

template <typename T, int DK>
struct SimtCfg {
  static constexpr int ROWS = 32;     // state rows per CTA
  static constexpr int THREADS = 128; // 4 lanes per row
  static constexpr int STAGE = 16;    // tokens per shared-memory stage
  static constexpr int CPL = DK / 4;  // columns per lane
  static constexpr int NV4 = CPL / 4;
  static constexpr int RAW_QK = STAGE * DK * (int)sizeof(T);
  static constexpr int RAW_V = STAGE * ROWS * (int)sizeof(T);
  static constexpr int RAW_BYTES = 2 * RAW_QK + RAW_V + 2 * STAGE * 4;
  static constexpr int F32_BYTES = (2 * STAGE * DK + STAGE * ROWS + 2 * STAGE) * 4;
  static constexpr int SMEM = 2 * RAW_BYTES + F32_BYTES;
  static_assert(RAW_QK % 16 == 0 && RAW_V % 16 == 0 && RAW_BYTES % 16 == 0, "alignment");
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(dst)), "l"(src));
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(dst)), "l"(src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;\n" ::); }

}  // namespace

template <typename T, typename TO, int DK>
__global__ void __launch_bounds__(128)
prefill_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                    const float *__restrict__ g, const float *__restrict__ beta,
                    const int32_t *__restrict__ cu, int N, long long Ttot, int Hqk, int Hv,
                    int DV, float scale, const void *s0, void *sfin, int state_bf16, int raw,
                    TO *__restrict__ o, int32_t *status) {
  using C = SimtCfg<T, DK>;
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned char *stage_buf[2] = {smem, smem + C::RAW_BYTES};
  float *fq = reinterpret_cast<float *>(smem + 2 * C::RAW_BYTES);
  float *fk = fq + C::STAGE * DK;
  float *fv = fk + C::STAGE * DK;
  float *fa = fv + C::STAGE * C::ROWS;
  float *fb = fa + C::STAGE;

  const int nslices = DV / C::ROWS;
  int unit = blockIdx.x;
  const int slice = unit % nslices;
  unit /= nslices;
  const int h = unit % Hv;
  const int n = unit / Hv;
  const int j = h / (Hv / Hqk);
  const int tid = threadIdx.x, r4 = tid & 3, rloc = tid >> 2;
  const int row = slice * C::ROWS + rloc;

  const long long c0 = cu[n], c1 = cu[n + 1];
  const bool bad = (c0 < 0) || (c1 < c0) || (c1 > Ttot) || (n == 0 && c0 != 0) ||
                   (n == N - 1 && c1 != Ttot);
  if (bad) {
    if (tid == 0) report_status(status, GDN_ERR_BAD_SEQLENS);
    return;
  }

  float S[C::CPL];
  const size_t srow = (((size_t)n * Hv + h) * DV + row) * DK;
#pragma unroll
  for (int m = 0; m < C::NV4; ++m) {
    if (s0) load_state4(s0, srow + 16 * m + 4 * r4, state_bf16, S + 4 * m);
    else S[4 * m] = S[4 * m + 1] = S[4 * m + 2] = S[4 * m + 3] = 0.f;
  }

  const long long L = c1 - c0;
  const int nstages = (int)((L + C::STAGE - 1) / C::STAGE);

  // Copy the raw inputs of stage s into raw buffer s % 2.
  auto issue = [&](int s) {
    unsigned char *buf = stage_buf[s & 1];
    const long long t0 = c0 + (long long)s * C::STAGE;
    const int cnt = (int)min((long long)C::STAGE, c1 - t0);
    constexpr int QK_CHUNKS = DK * (int)sizeof(T) / 16;  // 16-byte chunks per row
    constexpr int V_CHUNKS = C::ROWS * (int)sizeof(T) / 16;
    for (int idx = tid; idx < cnt * QK_CHUNKS; idx += C::THREADS) {
      const int t = idx / QK_CHUNKS, c = idx - t * QK_CHUNKS;
      const size_t src = ((size_t)(t0 + t) * Hqk + j) * DK * sizeof(T) + (size_t)c * 16;
      cp_async16(buf + t * DK * sizeof(T) + c * 16, reinterpret_cast<const unsigned char *>(q) + src);
      cp_async16(buf + C::RAW_QK + t * DK * sizeof(T) + c * 16,
                 reinterpret_cast<const unsigned char *>(k) + src);
    }
    for (int idx = tid; idx < cnt * V_CHUNKS; idx += C::THREADS) {
      const int t = idx / V_CHUNKS, c = idx - t * V_CHUNKS;
      const size_t src = (((size_t)(t0 + t) * Hv + h) * DV + slice * C::ROWS) * sizeof(T) + (size_t)c * 16;
      cp_async16(buf + 2 * C::RAW_QK + t * C::ROWS * sizeof(T) + c * 16,
                 reinterpret_cast<const unsigned char *>(v) + src);
    }
    if (tid < cnt) {
      float *gb = reinterpret_cast<float *>(buf + 2 * C::RAW_QK + C::RAW_V);
      cp_async4(gb + tid, g + (size_t)(t0 + tid) * Hv + h);
      cp_async4(gb + C::STAGE + tid, beta + (size_t)(t0 + tid) * Hv + h);
    }
  };

  if (nstages > 0) issue(0);
  cp_async_commit();
  for (int st = 0; st < nstages; ++st) {
    if (st + 1 < nstages) issue(st + 1);
    cp_async_commit();
    cp_async_wait_1();
    __syncthreads();

    const long long t0 = c0 + (long long)st * C::STAGE;
    const int cnt = (int)min((long long)C::STAGE, c1 - t0);
    {  // convert stage st to fp32
      const unsigned char *buf = stage_buf[st & 1];
      const T *rq = reinterpret_cast<const T *>(buf);
      const T *rk = reinterpret_cast<const T *>(buf + C::RAW_QK);
      const T *rv = reinterpret_cast<const T *>(buf + 2 * C::RAW_QK);
      const float *rg = reinterpret_cast<const float *>(buf + 2 * C::RAW_QK + C::RAW_V);
      for (int idx = tid * 4; idx < cnt * DK; idx += C::THREADS * 4) {
        float x[4];
        load4(rq + idx, x);
        *reinterpret_cast<float4 *>(fq + idx) = make_float4(x[0], x[1], x[2], x[3]);
        load4(rk + idx, x);
        *reinterpret_cast<float4 *>(fk + idx) = make_float4(x[0], x[1], x[2], x[3]);
      }
      for (int idx = tid * 4; idx < cnt * C::ROWS; idx += C::THREADS * 4) {
        float x[4];
        load4(rv + idx, x);
        *reinterpret_cast<float4 *>(fv + idx) = make_float4(x[0], x[1], x[2], x[3]);
      }
      if (tid < cnt) {
        fa[tid] = raw ? alpha_raw(rg[tid]) : expf(rg[tid]);
        fb[tid] = raw ? beta_raw(rg[C::STAGE + tid]) : rg[C::STAGE + tid];
      }
    }
    __syncthreads();
    if (raw) {  // unit L2 norm per token for k and q, one token per warp in turn
      const int warp = tid >> 5, lane = tid & 31;
      for (int t = warp; t < cnt; t += C::THREADS / 32) {
        float sk = 0.f, sq = 0.f;
        for (int d = lane; d < DK; d += 32) {
          sk = fmaf(fk[t * DK + d], fk[t * DK + d], sk);
          sq = fmaf(fq[t * DK + d], fq[t * DK + d], sq);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          sk += __shfl_xor_sync(0xffffffffu, sk, off);
          sq += __shfl_xor_sync(0xffffffffu, sq, off);
        }
        const float rk = inv_norm(sk), rq = inv_norm(sq);
        for (int d = lane; d < DK; d += 32) {
          fk[t * DK + d] *= rk;
          fq[t * DK + d] *= rq;
        }
      }
      __syncthreads();
    }

    for (int t = 0; t < cnt; ++t) {
      const float *kt = fk + t * DK;
      const float *qt = fq + t * DK;
      float u = 0.f;
      float kk[C::CPL];
#pragma unroll
      for (int m = 0; m < C::NV4; ++m) {
        const float4 x = *reinterpret_cast<const float4 *>(kt + 16 * m + 4 * r4);
        kk[4 * m + 0] = x.x; kk[4 * m + 1] = x.y; kk[4 * m + 2] = x.z; kk[4 * m + 3] = x.w;
      }
#pragma unroll
      for (int x = 0; x < C::CPL; ++x) u = fmaf(S[x], kk[x], u);
      u += __shfl_xor_sync(0xffffffffu, u, 1);
      u += __shfl_xor_sync(0xffffffffu, u, 2);
      const float a = fa[t];
      const float w = fb[t] * (fv[t * C::ROWS + rloc] - a * u);
#pragma unroll
      for (int x = 0; x < C::CPL; ++x) S[x] = fmaf(a, S[x], w * kk[x]);
      float p = 0.f;
#pragma unroll
      for (int m = 0; m < C::NV4; ++m) {
        const float4 x = *reinterpret_cast<const float4 *>(qt + 16 * m + 4 * r4);
        p = fmaf(S[4 * m + 0], x.x, p);
        p = fmaf(S[4 * m + 1], x.y, p);
        p = fmaf(S[4 * m + 2], x.z, p);
        p = fmaf(S[4 * m + 3], x.w, p);
      }
      p += __shfl_xor_sync(0xffffffffu, p, 1);
      p += __shfl_xor_sync(0xffffffffu, p, 2);
      if (r4 == 0) o[((size_t)(t0 + t) * Hv + h) * DV + row] = from_f32<TO>(scale * p);
    }
  }

  if (sfin) {
#pragma unroll
    for (int m = 0; m < C::NV4; ++m) store_state4(sfin, srow + 16 * m + 4 * r4, state_bf16, S + 4 * m);
  }
}

template <typename T, typename TO, int DK>
static cudaError_t launch_simt_t(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const int32_t *cu, int N, long long T_,
                                 int Hqk, int Hv, int Dv, float scale, const void *s0,
                                 void *sfin, int state_bf16, int raw, void *o, int32_t *status,
                                 cudaStream_t stream) {
  using C = SimtCfg<T, DK>;
  auto kern = prefill_simt_kernel<T, TO, DK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const unsigned blocks = (unsigned)N * (unsigned)Hv * (unsigned)(Dv / C::ROWS);
  kern<<<blocks, C::THREADS, C::SMEM, stream>>>(
      static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), g, beta,
      cu, N, T_, Hqk, Hv, Dv, scale, s0, sfin, state_bf16, raw, static_cast<TO *>(o), status);
  return cudaGetLastError();
}

cudaError_t launch_prefill_simt(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, const int32_t *cu, int N, long long T_,
                                int Hqk, int Hv, int Dk, int Dv, int dtype, int o_dtype,
                                int state_dtype, int input_form, float scale, const void *s0,
                                void *sfin, void *o, int32_t *status, cudaStream_t stream) {
  const int sb = state_dtype == GDN_DTYPE_BF16, raw = input_form == GDN_INPUT_RAW;
  return dispatch_types(dtype, o_dtype, [&](auto t, auto to) {
    using T = decltype(t);
    using TO = decltype(to);
    if (Dk == 128)
      return launch_simt_t<T, TO, 128>(q, k, v, g, beta, cu, N, T_, Hqk, Hv, Dv, scale, s0, sfin, sb, raw, o, status, stream);
    return launch_simt_t<T, TO, 64>(q, k, v, g, beta, cu, N, T_, Hqk, Hv, Dv, scale, s0, sfin, sb, raw, o, status, stream);
  });
}

}  // namespace gdn
