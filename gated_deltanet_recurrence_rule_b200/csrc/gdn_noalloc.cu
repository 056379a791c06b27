// gdn_noalloc.cu -- gdn_prefill_noalloc: the prefill entry point for callers
// that cannot allocate device memory.
//
// gdn_prefill needs a device workspace: at least its status header (then the
// bf16 head-dim-128 case runs the single-pass kernel), more for the faster
// two-phase kernels.  Some callers cannot call cudaMalloc to get one: code that runs
// where the device allocator belongs to someone else (a framework's caching
// allocator, a serving runtime's memory pool), real-time paths that must not
// take cudaMalloc's implicit device-wide synchronisation, and plugins that are
// only handed input and output buffers.  For them this file keeps the
// workspace in a file-scope __device__ array that lives as long as the library
// is loaded, and passes it to the unchanged gdn_prefill.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "gdn.h"
#include "gdn_common.cuh"

namespace gdn {
size_t prefill_min_workspace_bytes(int32_t num_seqs, int64_t total_tokens, int32_t Hqk, int32_t Hv,
                                   int32_t Dk, int32_t Dv, int32_t dtype);
}  // namespace gdn

namespace {

// Every GPU that loads the library holds this array until the process exits.
// It is exactly the workspace header (status word, wait limit, scheduler
// counters): the most gdn_prefill_noalloc ever needs, because with no more
// workspace than that gdn_prefill runs its single-pass kernels.
constexpr size_t kScratchBytes = gdn::kWorkspaceHeaderBytes;
static_assert(kScratchBytes >= gdn::kWorkspaceHeaderBytes, "the scratch holds the workspace header");
static __device__ __align__(256) unsigned char g_prefill_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_prefill_scratch on the current device, resolved once per
// device (host code must not use the symbol itself as an address).
int32_t scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_prefill_scratch) != cudaSuccess || !p) return GDN_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return GDN_OK;
}

}  // namespace

extern "C" int32_t gdn_prefill_noalloc(const void *q, const void *k, const void *v, const float *g,
                                       const float *beta, const int32_t *cu_seqlens,
                                       int32_t num_seqs, int64_t total_tokens,
                                       int32_t num_qk_heads, int32_t num_v_heads,
                                       int32_t head_dim_k, int32_t head_dim_v, int32_t dtype,
                                       int32_t o_dtype, float scale, const float *initial_state,
                                       float *final_state, void *o, int32_t *device_status,
                                       void *stream) {
  const size_t need = gdn::prefill_min_workspace_bytes(num_seqs, total_tokens, num_qk_heads,
                                                       num_v_heads, head_dim_k, head_dim_v, dtype);
  if (need > kScratchBytes) return GDN_ERR_WORKSPACE;  // beyond the built-in scratch
  void *scratch = nullptr;
  const int32_t st = scratch_address(&scratch);
  if (st != GDN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The scratch keeps the previous call's contents: its header (status word,
  // wait limit and scheduler counters) must start every call at zero.
  if (cudaMemsetAsync(scratch, 0, gdn::kWorkspaceHeaderBytes, s) != cudaSuccess) return GDN_ERR_CUDA;
  const int32_t rc = gdn_prefill(q, k, v, g, beta, cu_seqlens, num_seqs, total_tokens,
                                 num_qk_heads, num_v_heads, head_dim_k, head_dim_v, dtype,
                                 o_dtype, GDN_DTYPE_FP32, GDN_INPUT_PREPARED, scale, initial_state,
                                 final_state, o,
                                 scratch, kScratchBytes, stream);
  if (rc != GDN_OK) return rc;
  if (device_status &&
      cudaMemcpyAsync(device_status, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) !=
          cudaSuccess)
    return GDN_ERR_CUDA;
  return GDN_OK;
}
