// gdn_common.cuh -- small device helpers shared by the libgdn kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "gdn.h"

namespace gdn {

// Workspace header written by gdn_prefill (first 256 bytes of the workspace).
struct WorkspaceHeader {
  int32_t status;         // GDN_OK or a device-detected error code (first one wins)
  uint32_t wait_limit_us; // bounded-wait limit of the kernels in microseconds; 0 = 2 s
  uint32_t next_unit;     // dynamic work counter of persistent kernels
  uint32_t reserved1;
};
constexpr size_t kWorkspaceHeaderBytes = 256;

__device__ __forceinline__ void report_status(int32_t *status, int32_t code) {
  if (status) atomicCAS(status, GDN_OK, code);
}

// The wait limit the caller left in the workspace header (`status` is the
// workspace base), in microseconds; 0 means the default of 2 s.
__device__ __forceinline__ uint32_t header_wait_limit_us(const int32_t *status) {
  return status ? reinterpret_cast<const volatile WorkspaceHeader *>(status)->wait_limit_us : 0u;
}

// ---- element conversion ---------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Load 4 consecutive elements (8-byte aligned for bf16, 16-byte for fp32).
__device__ __forceinline__ void load4(const float *p, float out[4]) {
  const float4 x = *reinterpret_cast<const float4 *>(p);
  out[0] = x.x; out[1] = x.y; out[2] = x.z; out[3] = x.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float out[4]) {
  const uint2 x = *reinterpret_cast<const uint2 *>(p);
  out[0] = __uint_as_float(x.x << 16);
  out[1] = __uint_as_float(x.x & 0xffff0000u);
  out[2] = __uint_as_float(x.y << 16);
  out[3] = __uint_as_float(x.y & 0xffff0000u);
}

// States of the caller kept in fp32 or, at rest, in bf16 (widened exactly on
// load, rounded to nearest even on store).  `e` is an element index, a
// multiple of 4; the base pointer is 16-byte aligned.
__device__ __forceinline__ void load_state4(const void *base, size_t e, bool bf16, float out[4]) {
  if (bf16) load4(static_cast<const __nv_bfloat16 *>(base) + e, out);
  else load4(static_cast<const float *>(base) + e, out);
}
__device__ __forceinline__ void store_state4(void *base, size_t e, bool bf16, const float in[4]) {
  if (bf16) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(in[0], in[1]);
    const __nv_bfloat162 b = __floats2bfloat162_rn(in[2], in[3]);
    *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(base) + e) =
        make_uint2(*reinterpret_cast<const uint32_t *>(&a), *reinterpret_cast<const uint32_t *>(&b));
  } else {
    *reinterpret_cast<float4 *>(static_cast<float *>(base) + e) = make_float4(in[0], in[1], in[2], in[3]);
  }
}

// Gates from raw inputs (GDN_INPUT_RAW): log alpha = -softplus(a), written
// without overflow; alpha itself = e^{-softplus(a)} = 1 / (1 + e^a); beta =
// sigmoid(b).  Large |a|, |b| saturate to the limits 0 and 1.
__device__ __forceinline__ float log_alpha_raw(float a) {
  return -(fmaxf(a, 0.f) + log1pf(expf(-fabsf(a))));
}
__device__ __forceinline__ float alpha_raw(float a) { return 1.f / (1.f + expf(a)); }
__device__ __forceinline__ float beta_raw(float b) { return 1.f / (1.f + expf(-b)); }
// 1 / |x| from the sum of squares, 0 for a zero row (which then stays zero).
__device__ __forceinline__ float inv_norm(float ss) { return ss > 0.f ? 1.f / sqrtf(ss) : 0.f; }

// Streaming (evict-first) 128-bit global load / store for data touched once.
__device__ __forceinline__ float4 ld_stream(const float4 *p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(float4 *p, float4 v) { __stcs(p, v); }

// Call f(T{}, TO{}) with the input element type T (dtype) and output element
// type TO (o_dtype) as type tags.
template <class F>
__host__ auto dispatch_types(int dtype, int o_dtype, F &&f) {
  if (dtype == GDN_DTYPE_BF16) {
    if (o_dtype == GDN_DTYPE_BF16) return f(__nv_bfloat16{}, __nv_bfloat16{});
    return f(__nv_bfloat16{}, float{});
  }
  if (o_dtype == GDN_DTYPE_BF16) return f(float{}, __nv_bfloat16{});
  return f(float{}, float{});
}

// ---- host-side caches ----------------------------------------------------------
// A kernel's dynamic shared memory limit is set once per device (the attribute
// persists); later calls skip the runtime call.  `flags` is one static array
// per kernel, indexed by device.
template <typename K>
__host__ cudaError_t set_smem_once(K kernel, int bytes, std::atomic<bool> (&flags)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && flags[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) flags[dev].store(true, std::memory_order_release);
  return e;
}
// Multiprocessor count of the current device, queried once per device.
__host__ inline int sm_count() {
  static std::atomic<int> counts[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = counts[dev].load(std::memory_order_acquire);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    counts[dev].store(n, std::memory_order_release);
  }
  return n;
}

// ---- programmatic dependent launch ------------------------------------------
// Kernels launched with launch_pdl may be scheduled while the previous kernel
// on the stream is still finishing.  Each of them calls pdl_wait() before its
// first global memory access: that waits until the previous grid has completed
// and its writes are visible (a no-op when the kernel was launched normally),
// so only launch latency and block scheduling overlap the previous kernel's
// tail.  pdl_allow_next() lets the next such kernel be scheduled once every
// block of this grid has started.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_allow_next() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
__host__ cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                cudaStream_t stream, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace gdn
