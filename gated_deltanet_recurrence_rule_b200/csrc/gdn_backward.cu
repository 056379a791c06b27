// gdn_backward.cu -- backward pass of the gated delta rule (training), on CUDA
// cores in fp32.
//
// The forward rule is the one of "Inside Qwen3.8-27B: Hybrid DeltaNet
// Architecture, 256k Context, and 24GB Local Serving", section "Gated DeltaNet
// Mechanics" (the page's note says the block form serves training too); per
// (sequence, value head), with u = S_{t-1} k_t and w = v_t - alpha_t u,
//   S_t = alpha_t S_{t-1} + beta_t w k_t^T,   o_t = scale S_t q_t.
// Given dO = dL/do and dS = dL/dS_final, the chain rule runs backwards over
// the tokens with G = dL/dS_t:
//   G      += scale dO_t q_t^T
//   dq_t    = scale S_t^T dO_t
//   dv_t    = beta_t G k_t
//   dbeta_t = w . (G k_t)
//   dg_t    = alpha_t (<G, S_{t-1}> - beta_t (G k_t) . u)
//   dk_t    = beta_t G^T w - alpha_t beta_t S_{t-1}^T (G k_t)
//   G      <- alpha_t (G - beta_t (G k_t) k_t^T)
// and dS0 = G at the start of the sequence.
//
// Rows of S (and of G) evolve independently, so one CTA takes a slice of
// ROWS rows of one (sequence, value head): 4 lanes per state row, each lane
// holding Dk/4 columns of S and of G in registers.  Slices are chosen so that
// a small batch still fills the GPU (backward_slices); sums over the rows
// (dq, dk, dg, dbeta) are written per slice and added by a second kernel.
// Per CTA:
//   pass 1  forward from S0, storing a checkpoint of S every C tokens;
//   pass 2  chunks last to first: the chunk's states S_{t-1} are recomputed
//           from its checkpoint into a per-CTA scratch, then walked backwards.
// S^T x products (dq, dk) are column sums over all rows: a recursive-halving
// shuffle over the 8 rows of a warp, then a sum over warps in shared memory
// (double-buffered, one block barrier per token).  The partial sums are added
// in a fixed order by the second kernel, so the result does not depend on
// scheduling.
#include <algorithm>

#include "gdn_common.cuh"

namespace gdn {
namespace bwd {

constexpr int C = 16;  // tokens per checkpoint chunk

template <int DK, int ROWS, int LPR>
struct Cfg {
  static constexpr int THREADS = LPR * ROWS;  // LPR lanes per state row
  static constexpr int CPL = DK / LPR;        // columns per lane: 4 LPR m + 4 r + (0..3)
  static constexpr int NV4 = CPL / 4;
  static constexpr int NW = THREADS / 32;
  static constexpr int RPW = 32 / LPR;        // rows per warp
  static constexpr int KEEP = CPL / RPW;      // columns a lane keeps after the row halving
  // shared memory (floats)
  static constexpr int S_Q = 0, S_K = S_Q + C * DK, S_V = S_K + C * DK, S_DO = S_V + C * ROWS;
  static constexpr int S_A = S_DO + C * ROWS, S_B = S_A + C;
  static constexpr int S_RED = S_B + C;                  // [2 buffers][2 vectors][NW][DK]
  static constexpr int S_RS = S_RED + 2 * 2 * NW * DK;   // [2 buffers][3][NW]
  static constexpr int S_BASE = S_RS + 2 * 3 * NW;       // chunk base (int)
  static constexpr int FLOATS = S_BASE + 4;
  static constexpr size_t SMEM = FLOATS * sizeof(float);
};

struct Params {
  const void *q, *k, *v;
  const float *g, *beta;
  const int32_t *cu;
  int N, T, Hqk, Hv, Dv, R;  // R slices of Dv / R rows per (sequence, value head)
  float scale;
  const float *s0, *dO, *dSfin;
  float *dq, *dk;     // [T, Hv R, DK] per slice (the outputs themselves when Hv R == Hqk)
  float *dg, *dbeta;  // [T, Hv R] per slice (the outputs themselves when R == 1)
  float *dv, *ds0;
  float *ckpt;     // [(ceil(T / C) + N) * Hv][Dv x Dk states]
  float *scratch;  // [N * Hv * R][C states of a slice]
  int32_t *status;
};

// Column c = 4 LPR m + 4 r + q of this lane's row (r = lane % LPR), element
// e = 4 m + q.  Sum v over the 32 / LPR rows a warp holds (lane bits log2(LPR)
// .. 4) by recursive halving: at each level a lane keeps half of its elements
// and adds the partner's copy of them, so afterwards it holds CPL / (32 / LPR)
// consecutive elements (from keep_e0) summed over the warp's rows, with far
// fewer shuffles than one reduction per element.
template <int CPL, int LPR>
__device__ __forceinline__ void halve_rows(float (&v)[CPL], int lane) {
  int width = CPL;
#pragma unroll
  for (int b = 16; b >= LPR; b >>= 1) {
    width >>= 1;
    const bool up = lane & b;
#pragma unroll
    for (int e = 0; e < CPL / 2; ++e) {
      if (e < width) {
        const float mine = up ? v[width + e] : v[e], other = up ? v[e] : v[width + e];
        v[e] = mine + __shfl_xor_sync(0xffffffffu, other, b);
      }
    }
  }
}
// First element index (4 m + q) a lane keeps after halve_rows.
template <int CPL, int LPR>
__device__ __forceinline__ int keep_e0(int lane) {
  int e0 = 0, width = CPL;
#pragma unroll
  for (int b = 16; b >= LPR; b >>= 1) {
    width >>= 1;
    if (lane & b) e0 += width;
  }
  return e0;
}

template <typename T, int DK, int ROWS, int LPR>
__global__ void __launch_bounds__(LPR * ROWS, LPR * ROWS >= 512 ? 1 : 2)
backward_kernel(const Params p) {
  using CF = Cfg<DK, ROWS, LPR>;
  constexpr int CPL = CF::CPL, NV4 = CF::NV4, NW = CF::NW, KEEP = CF::KEEP;
  constexpr int CS = 4 * LPR;  // column stride between a lane's float4s
  extern __shared__ __align__(16) float sm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = tid / LPR, r4 = tid % LPR;  // row within the slice, lane within the row
  const int unit = blockIdx.x / p.R, slice = blockIdx.x - unit * p.R;
  const int n = unit / p.Hv, h = unit - n * p.Hv;
  const int j = h / (p.Hv / p.Hqk);
  const int DV = p.Dv, rowg = slice * ROWS + row;  // row within the head
  const int slot = h * p.R + slice;                // partial-sum slot of this CTA

  const int c0 = p.cu[n], c1 = p.cu[n + 1];
  if (c0 < 0 || c1 < c0 || c1 > p.T || (n == 0 && c0 != 0) || (n == p.N - 1 && c1 != p.T)) {
    if (tid == 0) report_status(p.status, GDN_ERR_BAD_SEQLENS);
    return;
  }
  const int L = c1 - c0, nck = (L + C - 1) / C;
  if (tid == 0) {  // first checkpoint of this sequence: chunks of the earlier sequences
    int base = 0;
    for (int m = 0; m < n; ++m) base += (p.cu[m + 1] - p.cu[m] + C - 1) / C;
    reinterpret_cast<int *>(sm + CF::S_BASE)[0] = base;
  }
  __syncthreads();
  const int cbase = reinterpret_cast<const int *>(sm + CF::S_BASE)[0];
  const size_t hs = (size_t)DV * DK, ss = (size_t)ROWS * DK;  // a head's / a slice's state
  const size_t srow = ((size_t)n * p.Hv + h) * hs + (size_t)rowg * DK;
  auto ck = [&](int c) {  // this thread's float4s of checkpoint c, laid out [NV4][THREADS]
    return reinterpret_cast<float4 *>(p.ckpt + ((size_t)(cbase + c) * p.Hv + h) * hs + slice * ss) + tid;
  };
  float4 *scr = reinterpret_cast<float4 *>(p.scratch + (size_t)blockIdx.x * C * ss) + tid;

  float *sq = sm + CF::S_Q, *sk = sm + CF::S_K, *sv = sm + CF::S_V, *sdo = sm + CF::S_DO;
  float *sa = sm + CF::S_A, *sb = sm + CF::S_B;
  // stage chunk c: k (and q, dO when `full`), v, alpha, beta as fp32
  auto stage = [&](int c, bool full) {
    const int t0 = c0 + c * C, cnt = min(C, c1 - t0);
    __syncthreads();  // the previous chunk's tokens are no longer read
    for (int x = tid; x < cnt * DK; x += CF::THREADS) {
      const int t = x / DK, d = x - t * DK;
      const size_t off = ((size_t)(t0 + t) * p.Hqk + j) * DK + d;
      sk[x] = to_f32(static_cast<const T *>(p.k)[off]);
      if (full) sq[x] = to_f32(static_cast<const T *>(p.q)[off]);
    }
    for (int x = tid; x < cnt * ROWS; x += CF::THREADS) {
      const int t = x / ROWS, d = x - t * ROWS;
      const size_t off = ((size_t)(t0 + t) * p.Hv + h) * DV + slice * ROWS + d;
      sv[x] = to_f32(static_cast<const T *>(p.v)[off]);
      if (full) sdo[x] = p.dO[off];
    }
    if (tid < cnt) {
      sa[tid] = expf(p.g[(size_t)(t0 + tid) * p.Hv + h]);
      sb[tid] = p.beta[(size_t)(t0 + tid) * p.Hv + h];
    }
    __syncthreads();
    return cnt;
  };
  auto rowdot = [&](const float (&x)[CPL], const float *vec) {  // (x . vec) over the row
    float a = 0.f;
#pragma unroll
    for (int m = 0; m < NV4; ++m) {
      const float4 y = *reinterpret_cast<const float4 *>(vec + CS * m + 4 * r4);
      a = fmaf(x[4 * m], y.x, a); a = fmaf(x[4 * m + 1], y.y, a);
      a = fmaf(x[4 * m + 2], y.z, a); a = fmaf(x[4 * m + 3], y.w, a);
    }
#pragma unroll
    for (int off = 1; off < LPR; off <<= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
    return a;
  };
  auto step = [&](float (&S)[CPL], int t) {  // S <- S_t from S_{t-1}
    const float *kt = sk + t * DK;
    const float u = rowdot(S, kt);
    const float w = sb[t] * (sv[t * ROWS + row] - sa[t] * u);
#pragma unroll
    for (int m = 0; m < NV4; ++m) {
      const float4 y = *reinterpret_cast<const float4 *>(kt + CS * m + 4 * r4);
      S[4 * m] = fmaf(sa[t], S[4 * m], w * y.x); S[4 * m + 1] = fmaf(sa[t], S[4 * m + 1], w * y.y);
      S[4 * m + 2] = fmaf(sa[t], S[4 * m + 2], w * y.z); S[4 * m + 3] = fmaf(sa[t], S[4 * m + 3], w * y.w);
    }
  };

  // ---- pass 1: forward with a checkpoint every C tokens
  float S[CPL];
#pragma unroll
  for (int m = 0; m < NV4; ++m) {
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p.s0) x = *reinterpret_cast<const float4 *>(p.s0 + srow + CS * m + 4 * r4);
    S[4 * m] = x.x; S[4 * m + 1] = x.y; S[4 * m + 2] = x.z; S[4 * m + 3] = x.w;
  }
  for (int c = 0; c < nck; ++c) {
    float4 *dst = ck(c);
#pragma unroll
    for (int m = 0; m < NV4; ++m)
      dst[m * CF::THREADS] = make_float4(S[4 * m], S[4 * m + 1], S[4 * m + 2], S[4 * m + 3]);
    const int cnt = stage(c, false);
    for (int t = 0; t < cnt; ++t) step(S, t);
  }

  // ---- pass 2: backwards
  float G[CPL];
#pragma unroll
  for (int m = 0; m < NV4; ++m) {
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p.dSfin) x = *reinterpret_cast<const float4 *>(p.dSfin + srow + CS * m + 4 * r4);
    G[4 * m] = x.x; G[4 * m + 1] = x.y; G[4 * m + 2] = x.z; G[4 * m + 3] = x.w;
  }
  float *red = sm + CF::S_RED, *rs = sm + CF::S_RS;
  int parity = 0;
  for (int c = nck - 1; c >= 0; --c) {
    const int cnt = stage(c, true);
    {  // S_{t-1} of every token of the chunk into the scratch
      const float4 *src = ck(c);
#pragma unroll
      for (int m = 0; m < NV4; ++m) {
        const float4 x = src[m * CF::THREADS];
        S[4 * m] = x.x; S[4 * m + 1] = x.y; S[4 * m + 2] = x.z; S[4 * m + 3] = x.w;
      }
      for (int t = 0; t < cnt; ++t) {
#pragma unroll
        for (int m = 0; m < NV4; ++m)
          scr[(t * NV4 + m) * CF::THREADS] = make_float4(S[4 * m], S[4 * m + 1], S[4 * m + 2], S[4 * m + 3]);
        if (t + 1 < cnt) step(S, t);
      }
    }
    for (int t = cnt - 1; t >= 0; --t) {
      const size_t tg = (size_t)(c0 + c * C + t);
      const float alpha = sa[t], bt = sb[t];
      const float *kt = sk + t * DK, *qt = sq + t * DK;
      float Sp[CPL];  // S_{t-1}
#pragma unroll
      for (int m = 0; m < NV4; ++m) {
        const float4 x = scr[(t * NV4 + m) * CF::THREADS];
        Sp[4 * m] = x.x; Sp[4 * m + 1] = x.y; Sp[4 * m + 2] = x.z; Sp[4 * m + 3] = x.w;
      }
      const float u = rowdot(Sp, kt);
      const float w = sv[t * ROWS + row] - alpha * u;  // v - alpha u (beta applied where used)
      const float sdO = p.scale * sdo[t * ROWS + row], bw = bt * w;
      float *rb = red + parity * 2 * NW * DK;
      const int e0 = keep_e0<CPL, LPR>(lane);
      float tmp[CPL];
      // G += scale dO q^T;  dq partial = scale dO_i S_t[i, :],  S_t = alpha S_{t-1} + beta w k^T
#pragma unroll
      for (int m = 0; m < NV4; ++m) {
        const float4 a = *reinterpret_cast<const float4 *>(kt + CS * m + 4 * r4);
        const float4 b = *reinterpret_cast<const float4 *>(qt + CS * m + 4 * r4);
        const float kk[4] = {a.x, a.y, a.z, a.w}, qq[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          G[4 * m + x] = fmaf(sdO, qq[x], G[4 * m + x]);
          tmp[4 * m + x] = sdO * fmaf(alpha, Sp[4 * m + x], bw * kk[x]);
        }
      }
      halve_rows<CPL, LPR>(tmp, lane);
#pragma unroll
      for (int x = 0; x < KEEP; ++x) {
        const int e = e0 + x;
        rb[warp * DK + CS * (e >> 2) + 4 * r4 + (e & 3)] = tmp[x];
      }
      float sgs = 0.f;
#pragma unroll
      for (int e = 0; e < CPL; ++e) sgs = fmaf(G[e], Sp[e], sgs);
      const float gk = rowdot(G, kt);
      // dk partial = beta w G[i, :] - alpha beta Gk_i S_{t-1}[i, :]
      const float abg = alpha * bt * gk;
#pragma unroll
      for (int e = 0; e < CPL; ++e) tmp[e] = fmaf(bw, G[e], -abg * Sp[e]);
      halve_rows<CPL, LPR>(tmp, lane);
#pragma unroll
      for (int x = 0; x < KEEP; ++x) {
        const int e = e0 + x;
        rb[NW * DK + warp * DK + CS * (e >> 2) + 4 * r4 + (e & 3)] = tmp[x];
      }
      if (r4 == 0) p.dv[(tg * p.Hv + h) * DV + rowg] = bt * gk;
      // scalars: <G, S_{t-1}> (every lane), (G k) . u and w . (G k) (one lane per row)
      float s3[3] = {sgs, r4 == 0 ? gk * u : 0.f, r4 == 0 ? w * gk : 0.f};
#pragma unroll
      for (int x = 0; x < 3; ++x)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s3[x] += __shfl_xor_sync(0xffffffffu, s3[x], off);
      if (lane == 0) {
        rs[parity * 3 * NW + warp] = s3[0];
        rs[parity * 3 * NW + NW + warp] = s3[1];
        rs[parity * 3 * NW + 2 * NW + warp] = s3[2];
      }
      // G <- alpha (G - beta (G k) k^T), before the barrier (registers only)
      const float bgk = bt * gk;
#pragma unroll
      for (int m = 0; m < NV4; ++m) {
        const float4 a = *reinterpret_cast<const float4 *>(kt + CS * m + 4 * r4);
        G[4 * m] = alpha * fmaf(-bgk, a.x, G[4 * m]);
        G[4 * m + 1] = alpha * fmaf(-bgk, a.y, G[4 * m + 1]);
        G[4 * m + 2] = alpha * fmaf(-bgk, a.z, G[4 * m + 2]);
        G[4 * m + 3] = alpha * fmaf(-bgk, a.w, G[4 * m + 3]);
      }
      __syncthreads();
      if (tid < DK) {
        float aq = 0.f, ak = 0.f;
#pragma unroll
        for (int x = 0; x < NW; ++x) {
          aq += rb[x * DK + tid];
          ak += rb[NW * DK + x * DK + tid];
        }
        p.dq[(tg * p.Hv * p.R + slot) * DK + tid] = aq;
        p.dk[(tg * p.Hv * p.R + slot) * DK + tid] = ak;
      }
      if (tid == 0) {  // (a block may have exactly DK threads)
        float a0 = 0.f, a1 = 0.f, a2 = 0.f;
#pragma unroll
        for (int x = 0; x < NW; ++x) {
          a0 += rs[parity * 3 * NW + x];
          a1 += rs[parity * 3 * NW + NW + x];
          a2 += rs[parity * 3 * NW + 2 * NW + x];
        }
        p.dg[tg * p.Hv * p.R + slot] = alpha * (a0 - bt * a1);  // linear in the row sums
        p.dbeta[tg * p.Hv * p.R + slot] = a2;
      }
      parity ^= 1;
    }
  }
  if (p.ds0) {
#pragma unroll
    for (int m = 0; m < NV4; ++m)
      *reinterpret_cast<float4 *>(p.ds0 + srow + CS * m + 4 * r4) =
          make_float4(G[4 * m], G[4 * m + 1], G[4 * m + 2], G[4 * m + 3]);
  }
}

// out[r][d] = sum over the `width` consecutive partial slots of group r:
// part is [rows * width][inner], out is [rows][inner] (dq, dk: a query/key
// head's value heads and slices; dg, dbeta: a value head's slices).
__global__ void group_sum_kernel(const float *__restrict__ part, float *__restrict__ out,
                                 size_t rows, int width, int inner) {
  const size_t total = rows * inner;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t r = i / inner, d = i - r * inner;
    const float *src = part + r * width * inner + d;
    float a = 0.f;
    for (int x = 0; x < width; ++x) a += src[(size_t)x * inner];
    out[i] = a;
  }
}

}  // namespace bwd

// Slices per (sequence, value head): doubled, down to 32 rows per CTA, until
// the grid has two CTAs per SM of a B200 (148 SMs).  A function of the sizes
// only, so the workspace query and the launch agree.
static int backward_slices(int64_t N, int Hv, int Dv) {
  int R = 1;
  while (Dv / (2 * R) >= 32 && N * Hv * R < 2 * 148) R *= 2;
  return R;
}

size_t backward_workspace_bytes(int64_t N, int64_t T, int Hqk, int Hv, int Dk, int Dv) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const int R = backward_slices(N, Hv, Dv);
  const size_t hs = (size_t)Dv * Dk * sizeof(float);
  size_t b = kWorkspaceHeaderBytes;
  b += up(((size_t)((T + bwd::C - 1) / bwd::C) + (size_t)N) * Hv * hs);  // checkpoints
  b += up((size_t)N * Hv * bwd::C * hs);                                  // per-CTA scratch
  if ((int64_t)Hv * R != Hqk) b += 2 * up((size_t)T * Hv * R * Dk * sizeof(float));  // dq, dk
  if (R > 1) b += 2 * up((size_t)T * Hv * R * sizeof(float));                        // dg, dbeta
  return b;
}

template <typename T, int DK, int ROWS>
static cudaError_t launch_bwd_t(const bwd::Params &prm, cudaStream_t stream) {
  // 8 lanes per row for slices of up to 64 rows (twice the warps of 4 lanes for
  // this latency-bound walk), 4 for whole 128-row heads (registers)
  constexpr int LPR = ROWS <= 64 ? 8 : 4;
  using CF = bwd::Cfg<DK, ROWS, LPR>;
  auto kern = bwd::backward_kernel<T, DK, ROWS, LPR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)CF::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)prm.N * (unsigned)prm.Hv * (unsigned)prm.R, CF::THREADS, CF::SMEM, stream>>>(prm);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_bwd_rows(const bwd::Params &prm, int Dk, int rows, cudaStream_t stream) {
  if (Dk == 128) {
    if (rows == 128) return launch_bwd_t<T, 128, 128>(prm, stream);
    if (rows == 64) return launch_bwd_t<T, 128, 64>(prm, stream);
    return launch_bwd_t<T, 128, 32>(prm, stream);
  }
  if (rows == 128) return launch_bwd_t<T, 64, 128>(prm, stream);
  if (rows == 64) return launch_bwd_t<T, 64, 64>(prm, stream);
  return launch_bwd_t<T, 64, 32>(prm, stream);
}

cudaError_t launch_backward(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const int32_t *cu, int N, long long T_, int Hqk,
                            int Hv, int Dk, int Dv, int dtype, float scale, const float *s0,
                            const float *dO, const float *dSfin, float *dq, float *dk, float *dv,
                            float *dg, float *dbeta, float *ds0, void *workspace,
                            cudaStream_t stream) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const int T = (int)T_;
  const int R = backward_slices(N, Hv, Dv);
  unsigned char *ws = static_cast<unsigned char *>(workspace);
  const size_t hs = (size_t)Dv * Dk * sizeof(float);
  bwd::Params prm;
  prm.q = q; prm.k = k; prm.v = v; prm.g = g; prm.beta = beta; prm.cu = cu;
  prm.N = N; prm.T = T; prm.Hqk = Hqk; prm.Hv = Hv; prm.Dv = Dv; prm.R = R; prm.scale = scale;
  prm.s0 = s0; prm.dO = dO; prm.dSfin = dSfin;
  prm.dv = dv; prm.ds0 = ds0;
  prm.status = reinterpret_cast<int32_t *>(ws);
  size_t off = kWorkspaceHeaderBytes;
  prm.ckpt = reinterpret_cast<float *>(ws + off);
  off += up(((size_t)((T + bwd::C - 1) / bwd::C) + (size_t)N) * Hv * hs);
  prm.scratch = reinterpret_cast<float *>(ws + off);
  off += up((size_t)N * Hv * bwd::C * hs);
  const bool qk_direct = (int64_t)Hv * R == Hqk, gb_direct = R == 1;
  prm.dq = dq; prm.dk = dk; prm.dg = dg; prm.dbeta = dbeta;
  if (!qk_direct) {
    prm.dq = reinterpret_cast<float *>(ws + off);
    off += up((size_t)T * Hv * R * Dk * sizeof(float));
    prm.dk = reinterpret_cast<float *>(ws + off);
    off += up((size_t)T * Hv * R * Dk * sizeof(float));
  }
  if (!gb_direct) {
    prm.dg = reinterpret_cast<float *>(ws + off);
    off += up((size_t)T * Hv * R * sizeof(float));
    prm.dbeta = reinterpret_cast<float *>(ws + off);
  }
  const int rows = Dv / R;
  cudaError_t e = dtype == GDN_DTYPE_BF16 ? launch_bwd_rows<__nv_bfloat16>(prm, Dk, rows, stream)
                                          : launch_bwd_rows<float>(prm, Dk, rows, stream);
  if (e != cudaSuccess || T == 0) return e;
  auto blocks = [](size_t total) { return (unsigned)std::min<size_t>((total + 255) / 256, 148 * 16); };
  if (!qk_direct) {
    const size_t rows_qk = (size_t)T * Hqk;
    const int width = Hv / Hqk * R;
    bwd::group_sum_kernel<<<blocks(rows_qk * Dk), 256, 0, stream>>>(prm.dq, dq, rows_qk, width, Dk);
    bwd::group_sum_kernel<<<blocks(rows_qk * Dk), 256, 0, stream>>>(prm.dk, dk, rows_qk, width, Dk);
  }
  if (!gb_direct) {
    const size_t rows_gb = (size_t)T * Hv;
    bwd::group_sum_kernel<<<blocks(rows_gb), 256, 0, stream>>>(prm.dg, dg, rows_gb, R, 1);
    bwd::group_sum_kernel<<<blocks(rows_gb), 256, 0, stream>>>(prm.dbeta, dbeta, rows_gb, R, 1);
  }
  return cudaGetLastError();
}

}  // namespace gdn
