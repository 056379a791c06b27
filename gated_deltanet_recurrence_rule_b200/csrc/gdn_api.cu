// gdn_api.cu -- the C ABI of libgdn.so (declared in include/gdn.h).
//
// Host-side argument validation, status codes and kernel dispatch.  No entry
// point allocates memory, keeps pointers between calls or synchronises,
// except gdn_get_device_status, which synchronises the stream it is given.
#include <algorithm>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn.h"
#include "gdn_common.cuh"

namespace gdn {
cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float *state, void *o, int B, int Hqk, int Hv,
                          int Dk, int Dv, int dtype, int o_dtype, float scale,
                          cudaStream_t stream);
cudaError_t launch_prefill_simt(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, const int32_t *cu, int N, long long T_,
                                int Hqk, int Hv, int Dk, int Dv, int dtype, int o_dtype,
                                int state_dtype, int input_form, float scale, const void *s0,
                                void *sfin, void *o, int32_t *status, cudaStream_t stream);
int decode_tokens_max();
cudaError_t launch_decode_tokens(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const void *state_in, void *state_out,
                                 const int32_t *src_slot, const int32_t *dst_slot, int num_slots,
                                 void *o, int B, int Tn, int Hqk, int Hv, int Dk, int Dv, int dtype,
                                 int o_dtype, int state_dtype, int input_form, float scale,
                                 int32_t *status, cudaStream_t s);
bool prefill_tc_supported(int Hqk, int Hv, int Dk, int Dv, int dtype);
cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const int32_t *cu, int N, long long T_, int Hqk,
                              int Hv, int o_dtype, int state_dtype, int input_form, float scale,
                              const void *s0, void *sfin, void *o, void *workspace,
                              cudaStream_t stream);
size_t twophase_workspace_bytes(int64_t N, int64_t T, int Hv);
size_t twophase_round_workspace_bytes(int64_t N, int Hv, int64_t chunks_per_round);
size_t twophase_min_workspace_bytes(int64_t N, int Hv);
int64_t twophase_launch_count(int64_t N, int64_t T, int Hv, size_t workspace_bytes);
cudaError_t launch_prefill_twophase(const void *q, const void *k, const void *v, const float *g,
                                    const float *beta, const int32_t *cu, int N, long long T_,
                                    int Hqk, int Hv, int o_dtype, int state_dtype, int input_form,
                                    float scale, const void *s0, void *sfin, void *o,
                                    void *workspace, size_t workspace_bytes, cudaStream_t stream);
size_t backward_workspace_bytes(int64_t N, int64_t T, int Hqk, int Hv, int Dk, int Dv);
size_t backward_chunked_workspace_bytes(int64_t N, int64_t T, int Hqk, int Hv, int Dk, int Dv);
cudaError_t launch_backward_chunked(const void *q, const void *k, const void *v, const float *g,
                                    const float *beta, const int32_t *cu, int N, long long T, int Hqk,
                                    int Hv, int Dk, int Dv, int dtype, float scale, const float *s0,
                                    const float *dO, const float *dSfin, float *dq, float *dk,
                                    float *dv, float *dg, float *dbeta, float *ds0, void *workspace,
                                    cudaStream_t stream);
cudaError_t launch_backward(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const int32_t *cu, int N, long long T_, int Hqk,
                            int Hv, int Dk, int Dv, int dtype, float scale, const float *s0,
                            const float *dO, const float *dSfin, float *dq, float *dk, float *dv,
                            float *dg, float *dbeta, float *ds0, void *workspace,
                            cudaStream_t stream);
}  // namespace gdn

namespace {

constexpr int32_t kVersion = 100;  // 0.1.0

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool dtype_ok(int32_t dtype) { return dtype == GDN_DTYPE_BF16 || dtype == GDN_DTYPE_FP32; }
bool form_ok(int32_t f) { return f == GDN_INPUT_PREPARED || f == GDN_INPUT_RAW; }

bool dims_ok(int32_t Hqk, int32_t Hv, int32_t Dk, int32_t Dv, int32_t dtype) {
  if (Hqk <= 0 || Hv <= 0 || Hv % Hqk != 0) return false;
  if (!dtype_ok(dtype)) return false;
  return Dk > 0 && Dv > 0;
}

bool dims_supported(int32_t Dk, int32_t Dv) {
  return (Dk == 64 || Dk == 128) && (Dv == 64 || Dv == 128);
}

int32_t cuda_status(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

}  // namespace

namespace gdn {
// Smallest workspace gdn_prefill accepts for these sizes (the status header;
// bf16 D=128 then runs the single-pass kernel), 0 for invalid sizes.
size_t prefill_min_workspace_bytes(int32_t num_seqs, int64_t total_tokens, int32_t Hqk, int32_t Hv,
                                   int32_t Dk, int32_t Dv, int32_t dtype) {
  if (num_seqs < 0 || total_tokens < 0 || !dims_ok(Hqk, Hv, Dk, Dv, dtype)) return 0;
  return kWorkspaceHeaderBytes;
}
}  // namespace gdn

extern "C" {

const char *gdn_status_string(int32_t status) {
  switch (status) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG: invalid argument";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: shape or dtype not supported";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA: a CUDA call or launch failed";
    case GDN_ERR_DEVICE_TIMEOUT: return "GDN_ERR_DEVICE_TIMEOUT: a bounded wait in a kernel ran out";
    case GDN_ERR_BAD_SEQLENS: return "GDN_ERR_BAD_SEQLENS: cu_seqlens is not 0 = c0 <= ... <= cN = T";
    case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE: workspace missing, misaligned or too small";
    default: return "GDN_ERR_UNKNOWN";
  }
}

int32_t gdn_version(void) { return kVersion; }

size_t gdn_prefill_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t num_qk_heads,
                                  int32_t num_v_heads, int32_t head_dim_k, int32_t head_dim_v,
                                  int32_t dtype) {
  if (num_seqs < 0 || total_tokens < 0) return 0;
  if (!dims_ok(num_qk_heads, num_v_heads, head_dim_k, head_dim_v, dtype)) return 0;
  if (gdn::prefill_tc_supported(num_qk_heads, num_v_heads, head_dim_k, head_dim_v, dtype))
    return gdn::twophase_workspace_bytes(num_seqs, total_tokens, num_v_heads);
  return gdn::kWorkspaceHeaderBytes;
}

size_t gdn_prefill_workspace_size_rounds(int32_t num_seqs, int64_t total_tokens,
                                         int32_t num_qk_heads, int32_t num_v_heads,
                                         int32_t head_dim_k, int32_t head_dim_v, int32_t dtype,
                                         int64_t chunks_per_round) {
  const size_t full = gdn_prefill_workspace_size(num_seqs, total_tokens, num_qk_heads, num_v_heads,
                                                 head_dim_k, head_dim_v, dtype);
  if (full == 0 || chunks_per_round < 0) return 0;
  if (chunks_per_round == 0 ||
      !gdn::prefill_tc_supported(num_qk_heads, num_v_heads, head_dim_k, head_dim_v, dtype))
    return full;
  const size_t r = gdn::twophase_round_workspace_bytes(num_seqs, num_v_heads, chunks_per_round);
  return r < full ? r : full;
}

int64_t gdn_prefill_launch_count(int32_t num_seqs, int64_t total_tokens, int32_t num_qk_heads,
                                 int32_t num_v_heads, int32_t head_dim_k, int32_t head_dim_v,
                                 int32_t dtype, size_t workspace_bytes) {
  if (num_seqs < 0 || total_tokens < 0 ||
      !dims_ok(num_qk_heads, num_v_heads, head_dim_k, head_dim_v, dtype))
    return -1;
  if (!dims_supported(head_dim_k, head_dim_v)) return -1;
  if (num_seqs == 0) return 0;
  if (workspace_bytes < gdn::kWorkspaceHeaderBytes) return -1;
  if (gdn::prefill_tc_supported(num_qk_heads, num_v_heads, head_dim_k, head_dim_v, dtype) &&
      workspace_bytes >= gdn::twophase_min_workspace_bytes(num_seqs, num_v_heads))
    return gdn::twophase_launch_count(num_seqs, total_tokens, num_v_heads, workspace_bytes);
  return 1;  // one single-pass kernel
}

int32_t gdn_prefill(const void *q, const void *k, const void *v, const float *g,
                    const float *beta, const int32_t *cu_seqlens, int32_t num_seqs,
                    int64_t total_tokens, int32_t num_qk_heads, int32_t num_v_heads,
                    int32_t head_dim_k, int32_t head_dim_v, int32_t dtype, int32_t o_dtype,
                    int32_t state_dtype, int32_t input_form, float scale,
                    const void *initial_state, void *final_state, void *o, void *workspace,
                    size_t workspace_bytes, void *stream) {
  if (num_seqs < 0 || total_tokens < 0 || total_tokens > INT32_MAX) return GDN_ERR_INVALID_ARG;
  if (!dims_ok(num_qk_heads, num_v_heads, head_dim_k, head_dim_v, dtype)) return GDN_ERR_INVALID_ARG;
  if (!dtype_ok(o_dtype) || !dtype_ok(state_dtype) || !form_ok(input_form)) return GDN_ERR_INVALID_ARG;
  if (!dims_supported(head_dim_k, head_dim_v)) return GDN_ERR_UNSUPPORTED;
  if (num_seqs == 0) return total_tokens == 0 ? GDN_OK : GDN_ERR_INVALID_ARG;
  if (!cu_seqlens || !aligned(cu_seqlens, 4)) return GDN_ERR_INVALID_ARG;
  if (total_tokens > 0) {
    if (!q || !k || !v || !g || !beta || !o) return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(g, 4) || !aligned(beta, 4))
      return GDN_ERR_INVALID_ARG;
  }
  if ((initial_state && !aligned(initial_state, 16)) || (final_state && !aligned(final_state, 16)))
    return GDN_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < gdn::kWorkspaceHeaderBytes)
    return GDN_ERR_WORKSPACE;
  // grid-size limits of the launches below
  if ((int64_t)num_seqs * num_v_heads * 4 > INT32_MAX) return GDN_ERR_UNSUPPORTED;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t *status = static_cast<int32_t *>(workspace);
  cudaError_t e;
  if (gdn::prefill_tc_supported(num_qk_heads, num_v_heads, head_dim_k, head_dim_v, dtype)) {
    if (workspace_bytes >= gdn::twophase_min_workspace_bytes(num_seqs, num_v_heads)) {
      // two phases: every chunk's state-free products at once, then the state pass
      e = gdn::launch_prefill_twophase(q, k, v, g, beta, cu_seqlens, num_seqs, total_tokens,
                                       num_qk_heads, num_v_heads, o_dtype, state_dtype, input_form,
                                       scale, initial_state, final_state, o, workspace,
                                       workspace_bytes, s);
    } else {
      // a header-only workspace: one pass, each CTA does all of a (sequence, head)
      e = gdn::launch_prefill_tc(q, k, v, g, beta, cu_seqlens, num_seqs, total_tokens,
                                 num_qk_heads, num_v_heads, o_dtype, state_dtype, input_form,
                                 scale, initial_state, final_state, o, workspace, s);
    }
  } else {
    e = gdn::launch_prefill_simt(q, k, v, g, beta, cu_seqlens, num_seqs, total_tokens,
                                 num_qk_heads, num_v_heads, head_dim_k, head_dim_v, dtype, o_dtype,
                                 state_dtype, input_form, scale, initial_state, final_state, o,
                                 status, s);
  }
  return cuda_status(e);
}

int32_t gdn_decode_step(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, float *state, void *o, int32_t batch,
                        int32_t num_qk_heads, int32_t num_v_heads, int32_t head_dim_k,
                        int32_t head_dim_v, int32_t dtype, int32_t o_dtype, float scale,
                        void *stream) {
  if (batch < 0) return GDN_ERR_INVALID_ARG;
  if (!dims_ok(num_qk_heads, num_v_heads, head_dim_k, head_dim_v, dtype)) return GDN_ERR_INVALID_ARG;
  if (!dtype_ok(o_dtype)) return GDN_ERR_INVALID_ARG;
  if (!dims_supported(head_dim_k, head_dim_v)) return GDN_ERR_UNSUPPORTED;
  if (batch == 0) return GDN_OK;
  if ((int64_t)batch * num_v_heads > INT32_MAX) return GDN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !g || !beta || !state || !o) return GDN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(state, 16) || !aligned(g, 4) || !aligned(beta, 4))
    return GDN_ERR_INVALID_ARG;
  return cuda_status(gdn::launch_decode(q, k, v, g, beta, state, o, batch, num_qk_heads,
                                        num_v_heads, head_dim_k, head_dim_v, dtype, o_dtype,
                                        scale, static_cast<cudaStream_t>(stream)));
}

int32_t gdn_decode_tokens(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const void *state_in, void *state_out,
                          const int32_t *src_slot, const int32_t *dst_slot, int32_t num_slots,
                          void *o, int32_t batch, int32_t tokens, int32_t num_qk_heads,
                          int32_t num_v_heads, int32_t head_dim_k, int32_t head_dim_v,
                          int32_t dtype, int32_t o_dtype, int32_t state_dtype,
                          int32_t input_form, float scale, int32_t *device_status, void *stream) {
  if (batch < 0 || tokens < 0 || num_slots < 0) return GDN_ERR_INVALID_ARG;
  if (!form_ok(input_form)) return GDN_ERR_INVALID_ARG;
  if (!dims_ok(num_qk_heads, num_v_heads, head_dim_k, head_dim_v, dtype)) return GDN_ERR_INVALID_ARG;
  if (!dtype_ok(o_dtype) || !dtype_ok(state_dtype)) return GDN_ERR_INVALID_ARG;
  if (!dims_supported(head_dim_k, head_dim_v)) return GDN_ERR_UNSUPPORTED;
  if (tokens > gdn::decode_tokens_max()) return GDN_ERR_UNSUPPORTED;
  if (batch == 0 || tokens == 0) return GDN_OK;
  if ((int64_t)batch * num_v_heads > INT32_MAX) return GDN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !g || !beta || !state_in || !state_out || !o) return GDN_ERR_INVALID_ARG;
  if (!src_slot && batch > num_slots) return GDN_ERR_INVALID_ARG;  // slot b for sequence b
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 4) ||
      !aligned(state_in, 16) || !aligned(state_out, 16) || !aligned(g, 4) || !aligned(beta, 4) ||
      (src_slot && !aligned(src_slot, 4)) || (dst_slot && !aligned(dst_slot, 4)) ||
      (device_status && !aligned(device_status, 4)))
    return GDN_ERR_INVALID_ARG;
  return cuda_status(gdn::launch_decode_tokens(
      q, k, v, g, beta, state_in, state_out, src_slot, dst_slot, num_slots, o, batch, tokens,
      num_qk_heads, num_v_heads, head_dim_k, head_dim_v, dtype, o_dtype, state_dtype, input_form,
      scale, device_status, static_cast<cudaStream_t>(stream)));
}

size_t gdn_prefill_backward_workspace_size(int32_t num_seqs, int64_t total_tokens,
                                           int32_t num_qk_heads, int32_t num_v_heads,
                                           int32_t head_dim_k, int32_t head_dim_v) {
  if (num_seqs < 0 || total_tokens < 0 || total_tokens > INT32_MAX) return 0;
  if (!dims_ok(num_qk_heads, num_v_heads, head_dim_k, head_dim_v, GDN_DTYPE_FP32)) return 0;
  if (!dims_supported(head_dim_k, head_dim_v)) return 0;
  return std::max(gdn::backward_chunked_workspace_bytes(num_seqs, total_tokens, num_qk_heads,
                                                        num_v_heads, head_dim_k, head_dim_v),
                  gdn::backward_workspace_bytes(num_seqs, total_tokens, num_qk_heads, num_v_heads,
                                                head_dim_k, head_dim_v));
}

size_t gdn_prefill_backward_workspace_size_sequential(int32_t num_seqs, int64_t total_tokens,
                                                      int32_t num_qk_heads, int32_t num_v_heads,
                                                      int32_t head_dim_k, int32_t head_dim_v) {
  if (num_seqs < 0 || total_tokens < 0 || total_tokens > INT32_MAX) return 0;
  if (!dims_ok(num_qk_heads, num_v_heads, head_dim_k, head_dim_v, GDN_DTYPE_FP32)) return 0;
  if (!dims_supported(head_dim_k, head_dim_v)) return 0;
  return gdn::backward_workspace_bytes(num_seqs, total_tokens, num_qk_heads, num_v_heads, head_dim_k,
                                       head_dim_v);
}

namespace {

constexpr int32_t kNothingToDo = -1;  // valid call with no sequences: return GDN_OK, launch nothing

// Host checks shared by both backward entry points: GDN_OK to proceed,
// kNothingToDo, or an error code.
int32_t check_backward(const void *q, const void *k, const void *v, const float *g,
                       const float *beta, const int32_t *cu_seqlens, int32_t num_seqs,
                       int64_t total_tokens, int32_t num_qk_heads, int32_t num_v_heads,
                       int32_t head_dim_k, int32_t head_dim_v, int32_t dtype,
                       const float *initial_state, const float *d_o, const float *d_final_state,
                       const float *dq, const float *dk, const float *dv, const float *dg,
                       const float *dbeta, const float *d_initial_state, const void *workspace) {
  if (num_seqs < 0 || total_tokens < 0 || total_tokens > INT32_MAX) return GDN_ERR_INVALID_ARG;
  if (!dims_ok(num_qk_heads, num_v_heads, head_dim_k, head_dim_v, dtype)) return GDN_ERR_INVALID_ARG;
  if (!dims_supported(head_dim_k, head_dim_v)) return GDN_ERR_UNSUPPORTED;
  if (num_seqs == 0) return total_tokens == 0 ? kNothingToDo : GDN_ERR_INVALID_ARG;
  if ((int64_t)num_seqs * num_v_heads > INT32_MAX) return GDN_ERR_UNSUPPORTED;
  if (!cu_seqlens || !aligned(cu_seqlens, 4)) return GDN_ERR_INVALID_ARG;
  if (total_tokens > 0) {
    if (!q || !k || !v || !g || !beta || !d_o || !dq || !dk || !dv || !dg || !dbeta)
      return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(d_o, 16) ||
        !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(g, 4) ||
        !aligned(beta, 4) || !aligned(dg, 4) || !aligned(dbeta, 4))
      return GDN_ERR_INVALID_ARG;
  }
  if ((initial_state && !aligned(initial_state, 16)) || (d_final_state && !aligned(d_final_state, 16)) ||
      (d_initial_state && !aligned(d_initial_state, 16)))
    return GDN_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256)) return GDN_ERR_WORKSPACE;
  return GDN_OK;
}

}  // namespace

int32_t gdn_prefill_backward(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const int32_t *cu_seqlens, int32_t num_seqs,
                             int64_t total_tokens, int32_t num_qk_heads, int32_t num_v_heads,
                             int32_t head_dim_k, int32_t head_dim_v, int32_t dtype, float scale,
                             const float *initial_state, const float *d_o,
                             const float *d_final_state, float *dq, float *dk, float *dv,
                             float *dg, float *dbeta, float *d_initial_state, void *workspace,
                             size_t workspace_bytes, void *stream) {
  const int32_t c = check_backward(q, k, v, g, beta, cu_seqlens, num_seqs, total_tokens, num_qk_heads,
                                   num_v_heads, head_dim_k, head_dim_v, dtype, initial_state, d_o,
                                   d_final_state, dq, dk, dv, dg, dbeta, d_initial_state, workspace);
  if (c != GDN_OK) return c == kNothingToDo ? GDN_OK : c;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (workspace_bytes >= gdn::backward_chunked_workspace_bytes(num_seqs, total_tokens, num_qk_heads,
                                                              num_v_heads, head_dim_k, head_dim_v))
    return cuda_status(gdn::launch_backward_chunked(
        q, k, v, g, beta, cu_seqlens, num_seqs, total_tokens, num_qk_heads, num_v_heads, head_dim_k,
        head_dim_v, dtype, scale, initial_state, d_o, d_final_state, dq, dk, dv, dg, dbeta,
        d_initial_state, workspace, st));
  if (workspace_bytes >= gdn::backward_workspace_bytes(num_seqs, total_tokens, num_qk_heads,
                                                       num_v_heads, head_dim_k, head_dim_v))
    return cuda_status(gdn::launch_backward(
        q, k, v, g, beta, cu_seqlens, num_seqs, total_tokens, num_qk_heads, num_v_heads, head_dim_k,
        head_dim_v, dtype, scale, initial_state, d_o, d_final_state, dq, dk, dv, dg, dbeta,
        d_initial_state, workspace, st));
  return GDN_ERR_WORKSPACE;
}

int32_t gdn_prefill_backward_sequential(const void *q, const void *k, const void *v, const float *g,
                                        const float *beta, const int32_t *cu_seqlens,
                                        int32_t num_seqs, int64_t total_tokens,
                                        int32_t num_qk_heads, int32_t num_v_heads,
                                        int32_t head_dim_k, int32_t head_dim_v, int32_t dtype,
                                        float scale, const float *initial_state, const float *d_o,
                                        const float *d_final_state, float *dq, float *dk,
                                        float *dv, float *dg, float *dbeta, float *d_initial_state,
                                        void *workspace, size_t workspace_bytes, void *stream) {
  const int32_t c = check_backward(q, k, v, g, beta, cu_seqlens, num_seqs, total_tokens, num_qk_heads,
                                   num_v_heads, head_dim_k, head_dim_v, dtype, initial_state, d_o,
                                   d_final_state, dq, dk, dv, dg, dbeta, d_initial_state, workspace);
  if (c != GDN_OK) return c == kNothingToDo ? GDN_OK : c;
  if (workspace_bytes < gdn::backward_workspace_bytes(num_seqs, total_tokens, num_qk_heads,
                                                      num_v_heads, head_dim_k, head_dim_v))
    return GDN_ERR_WORKSPACE;
  return cuda_status(gdn::launch_backward(
      q, k, v, g, beta, cu_seqlens, num_seqs, total_tokens, num_qk_heads, num_v_heads, head_dim_k,
      head_dim_v, dtype, scale, initial_state, d_o, d_final_state, dq, dk, dv, dg, dbeta,
      d_initial_state, workspace, static_cast<cudaStream_t>(stream)));
}

int32_t gdn_prefill_uses_tensor_cores(int32_t num_qk_heads, int32_t num_v_heads,
                                      int32_t head_dim_k, int32_t head_dim_v, int32_t dtype) {
  if (!dims_ok(num_qk_heads, num_v_heads, head_dim_k, head_dim_v, dtype)) return 0;
  return gdn::prefill_tc_supported(num_qk_heads, num_v_heads, head_dim_k, head_dim_v, dtype) ? 1 : 0;
}

int32_t gdn_get_device_status(const void *workspace, void *stream, int32_t *status_host) {
  if (!workspace || !status_host || !aligned(workspace, 256)) return GDN_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t value = GDN_OK;
  cudaError_t e = cudaMemcpyAsync(&value, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(const_cast<void *>(workspace), 0, sizeof(int32_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return GDN_ERR_CUDA;
  *status_host = value;
  return GDN_OK;
}

}  // extern "C"
