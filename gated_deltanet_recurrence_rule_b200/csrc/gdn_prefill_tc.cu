// gdn_prefill_tc.cu -- tensor-core (tcgen05) chunked prefill.  Not built yet:
// every prefill call takes the CUDA-core kernel.
#include "gdn_common.cuh"

namespace gdn {

bool prefill_tc_supported(int, int, int, int, int) { return false; }

cudaError_t launch_prefill_tc(const void *, const void *, const void *, const float *,
                              const float *, const int32_t *, int, long long, int, int, int, float,
                              const float *, float *, void *, void *, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace gdn
