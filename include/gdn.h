/*
 * gdn.h -- C ABI of libgdn.so: the Gated DeltaNet recurrence (gated delta
 * rule) on NVIDIA B200 (sm_100a).
 *
 * The operation.  For every sequence and every value head h, with state
 * S (Dv x Dk, fp32) and per-token decay alpha_t = exp(g_t) and write strength
 * beta_t:
 *
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = scale * S_t q_t
 *
 * Source: "Inside Qwen3.8-27B: Hybrid DeltaNet Architecture, 256k Context,
 * and 24GB Local Serving", section "Gated DeltaNet Mechanics" (the delta rule
 * subtracts the association stored under the normalized key k_t before
 * writing the value v_t; S_t is a fixed-size d x d state; prefill uses a
 * block-parallel chunked form, inference updates the state token by token).
 * Head layout: "Qwen 3.8 27B Review: Native Vision, FP8 Quantization & 1M
 * Context in a Compact Dense Model", section "3. Architecture: Gated DeltaNet
 * Hybrid + FP8 Quantization" (16 query/key heads, 48 value heads, head dim
 * 128).
 *
 * Conventions fixed by this library where the pages are silent:
 *   - State layout [num_seqs, Hv, Dv, Dk], fp32 (or bf16 at rest where a
 *     state_dtype says so), row i = value dim i, Dk contiguous.  Read u = S k,
 *     write v k^T, output S q.
 *   - Value head h reads query/key head h / (Hv / Hqk) (contiguous groups);
 *     Hv must be a multiple of Hqk.  No copies are made for the sharing.
 *   - g (= log alpha, <= 0) and beta are fp32, one per (token, value head).
 *   - o_t uses the state after token t.
 *   - q and k are used as given (the caller normalises them), unless an
 *     input_form of GDN_INPUT_RAW asks the kernels to do it.
 *
 * Memory.  Every pointer argument except those named "host" is a device
 * pointer (cudaMalloc'd or equivalent) owned by the caller; the library never
 * allocates device memory, frees or keeps a pointer after a call returns.  The
 * pipelined prefill (see gdn_prefill) keeps two internal streams and a few
 * events per (device, caller stream) for up to 8 caller streams per device,
 * created on first use and kept until the process exits; prefills issued on
 * further caller streams share the device's first pair and are then ordered
 * after one another (correct, but not concurrent).  All arrays are dense
 * row-major with the shapes given below and 16-byte-aligned bases.
 *
 * Ordering.  Every call enqueues work on `stream` (a cudaStream_t; NULL is
 * the legacy default stream) and returns without synchronising, except
 * gdn_get_device_status, which synchronises that stream.
 *
 * Errors.  Arguments are validated on the host before any launch; an invalid
 * call returns a nonzero status and enqueues nothing.  A failed launch
 * returns GDN_ERR_CUDA.  Conditions only the device can see (inconsistent
 * cu_seqlens contents, a bounded wait that ran out) are recorded in the
 * workspace status word; read them with gdn_get_device_status.  Nothing in
 * the library aborts, traps or throws.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes (returned as int32_t). */
#define GDN_OK 0
#define GDN_ERR_INVALID_ARG 1    /* null / misaligned pointer, bad size or dtype        */
#define GDN_ERR_UNSUPPORTED 2    /* valid but not implemented (head dims, dtype combo)  */
#define GDN_ERR_CUDA 3           /* a CUDA runtime call or launch failed                */
#define GDN_ERR_DEVICE_TIMEOUT 4 /* device status: a bounded wait inside a kernel ran out */
#define GDN_ERR_BAD_SEQLENS 5    /* device status: cu_seqlens not 0 = c0 <= c1 .. <= cN = T */
#define GDN_ERR_WORKSPACE 6      /* workspace missing, misaligned or too small           */

/* Element types of q, k, v (dtype), of o (o_dtype) and of the states kept
 * between calls (state_dtype, where an entry point takes one; fp32 elsewhere);
 * g and beta are always fp32.  o_dtype is chosen independently: fp32 o keeps
 * the precision the fp32 arithmetic carries (rounding o to bf16 alone costs up
 * to 2^-8 |o| per element). */
#define GDN_DTYPE_BF16 0
#define GDN_DTYPE_FP32 1

/* Form of the per-token inputs (input_form).
 *   GDN_INPUT_PREPARED  q and k L2-normalised by the caller, g = log alpha,
 *                       beta the write strength.
 *   GDN_INPUT_RAW       the layer's raw projections: the kernels normalise each
 *                       (token, query/key head) row of q and k to unit L2 norm
 *                       (a zero row stays zero), read g as a with
 *                       alpha = e^{-softplus(a)} = 1 / (1 + e^a), and beta as b
 *                       with beta = sigmoid(b).  No normalised copy is written.
 * "Inside Qwen3.8-27B ...", section "Gated DeltaNet Mechanics", calls k the
 * normalized key projection and makes beta input dependent; softplus and
 * sigmoid are the plainest maps to a decay and a write strength in (0, 1). */
#define GDN_INPUT_PREPARED 0
#define GDN_INPUT_RAW 1

/* Human-readable name of a status code (static string, never NULL). */
const char *gdn_status_string(int32_t status);

/* Library version: major * 10000 + minor * 100 + patch. */
int32_t gdn_version(void);

/*
 * Bytes of device workspace with which gdn_prefill runs at full speed for
 * these sizes.  The workspace holds the device status word and, for the
 * tensor-core path, the per-chunk products of its first phase (about 65 KiB
 * per chunk of 64 tokens and value head, plus 2 x Hv x 64 KiB of state
 * carry).  It must stay allocated and unused by anything else until the
 * call's work on the stream has finished.  Returns 0 for invalid sizes.
 */
size_t gdn_prefill_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t num_qk_heads,
                                  int32_t num_v_heads, int32_t head_dim_k, int32_t head_dim_v,
                                  int32_t dtype);

/*
 * Bytes of a workspace with which the tensor-core prefill processes the packed
 * chunk list in rounds of `chunks_per_round` chunks (of 64 tokens, across all
 * value heads): a bounded workspace for long inputs, at the price of one
 * launch pair per round.  0 means one round (= gdn_prefill_workspace_size);
 * sizes that need no rounds return gdn_prefill_workspace_size.  Returns 0 for
 * invalid sizes or a negative chunks_per_round.
 */
size_t gdn_prefill_workspace_size_rounds(int32_t num_seqs, int64_t total_tokens,
                                         int32_t num_qk_heads, int32_t num_v_heads,
                                         int32_t head_dim_k, int32_t head_dim_v, int32_t dtype,
                                         int64_t chunks_per_round);

/*
 * Number of kernel launches one gdn_prefill call with these sizes and this
 * workspace makes (0 for num_seqs = 0), or -1 for invalid arguments.  Host
 * only.  For sizing CUDA graphs and for counting launches in benchmarks.
 */
int64_t gdn_prefill_launch_count(int32_t num_seqs, int64_t total_tokens, int32_t num_qk_heads,
                                 int32_t num_v_heads, int32_t head_dim_k, int32_t head_dim_v,
                                 int32_t dtype, size_t workspace_bytes);

/*
 * Prefill: run the recurrence over num_seqs packed sequences.
 *
 * The chunked (block-parallel) form: "Inside Qwen3.8-27B ...", section "Gated
 * DeltaNet Mechanics" (the note that prefill is rewritten into a
 * block-parallel form for tensor cores with the state kept on chip).  Chunks
 * of 64 tokens aligned to each sequence's first token; the result equals the
 * token-by-token definition up to rounding.
 *
 *   q, k           [T, Hqk, Dk]   dtype
 *   v              [T, Hv, Dv]    dtype
 *   g, beta        [T, Hv]        fp32  (g = log alpha; -inf allowed: alpha = 0)
 *   cu_seqlens     [num_seqs + 1] int32, device; 0 = c_0 <= c_1 <= ... <= c_N = T.
 *                  Sequence n is tokens [c_n, c_{n+1}); empty sequences are allowed
 *                  (their final state equals their initial state).
 *   state_dtype    GDN_DTYPE_FP32, or GDN_DTYPE_BF16 for states kept at rest in
 *                  bf16: the initial state is widened exactly, the arithmetic is
 *                  the same as with fp32 states, and the final state is rounded
 *                  to nearest even once, when it is stored.
 *   input_form     GDN_INPUT_PREPARED or GDN_INPUT_RAW (see above): with raw
 *                  inputs q and k are normalised and g, beta mapped inside the
 *                  kernels (the tensor-core kernels fold 1/|q_t|, 1/|k_t| into
 *                  their per-token scalars; the bf16 operand tiles stay raw).
 *   initial_state  [num_seqs, Hv, Dv, Dk] state_dtype, or NULL for zeros.
 *   final_state    [num_seqs, Hv, Dv, Dk] state_dtype, or NULL to skip.  May be the
 *                  same pointer as initial_state (updated in place); no other
 *                  overlap between arguments is allowed.
 *   o              [T, Hv, Dv]    o_dtype (output)
 *   scale          multiplies o (1.0 for o_t = S_t q_t)
 *   workspace      device buffer of workspace_bytes >= 256 bytes, 256-byte aligned,
 *                  zero-filled once before its first use.  Its first word is the
 *                  sticky status word: it keeps the first device-detected error
 *                  until gdn_get_device_status reads and clears it.  Its second
 *                  word (uint32, byte offset 4) is the limit of the kernels'
 *                  bounded waits in microseconds, 0 for the default of 2 s; a
 *                  wait that runs out sets GDN_ERR_DEVICE_TIMEOUT, the kernel
 *                  drains its own copies and MMAs, frees its tensor memory and
 *                  returns, and o and final_state of that call are undefined
 *                  (tests set a limit of a microsecond to take that path).
 *                  Nothing else in it needs to survive between calls.
 *
 * Supported: Hv % Hqk == 0; Dk, Dv in {64, 128}; dtype and o_dtype each bf16
 * or fp32.  bf16 inputs with Dk = Dv = 128 run on the tensor cores (tcgen05,
 * bf16 operands with hi/lo splits of computed values, fp32 accumulation):
 *   - workspace_bytes >= gdn_prefill_workspace_size(...): two phases, the
 *     state-free products of every chunk at once (WY/UT transform), then one
 *     pass per (sequence, value head) over its chunks for the state, in
 *     pipelined rounds on the two internal streams of the caller's stream
 *     (joined to `stream` by events, so the call stays stream-ordered and can
 *     be captured in a CUDA graph);
 *   - smaller, down to the two-phase minimum (the state carry plus one chunk
 *     per value head): the same in rounds of as many chunks as fit;
 *   - below that (>= 256 bytes): a single-pass kernel, one CTA per (sequence,
 *     value head) doing all of each chunk in turn.  It is slower when the
 *     (sequence, value head) units do not fill the GPU several times over
 *     (one 8192-token sequence at 48 value heads: 1.29 ms against 0.56 ms),
 *     and faster when they do and no sequence is much longer than the rest
 *     (32 sequences of 1k to 32k tokens: 29.7 ms against 32.8 ms).  The host
 *     does not see the sequence lengths, so this choice is the caller's.
 * Every other case runs the fp32 CUDA-core kernel, which needs 256 bytes.
 * T = 0 or num_seqs = 0 is a valid no-op apart from copying initial_state to
 * final_state.
 */
int32_t gdn_prefill(const void *q, const void *k, const void *v, const float *g,
                    const float *beta, const int32_t *cu_seqlens, int32_t num_seqs,
                    int64_t total_tokens, int32_t num_qk_heads, int32_t num_v_heads,
                    int32_t head_dim_k, int32_t head_dim_v, int32_t dtype, int32_t o_dtype,
                    int32_t state_dtype, int32_t input_form, float scale,
                    const void *initial_state, void *final_state, void *o, void *workspace,
                    size_t workspace_bytes, void *stream);

/*
 * Prefill for callers that cannot allocate device memory.  (The pages have no
 * counterpart; this is a calling convention of the library.)  Some callers
 * cannot call cudaMalloc for gdn_prefill's workspace: the device allocator
 * belongs to someone else (a framework's caching allocator, a serving
 * runtime's memory pool), the path is real-time and must not take
 * cudaMalloc's implicit device-wide synchronisation, or a plugin is handed
 * only its input and output buffers.  This entry point allocates nothing: it
 * runs gdn_prefill with a 256-byte workspace (the status header) kept in a
 * file-scope __device__ array of the library (every GPU that loads the
 * library holds it until the process exits), and calls no cudaMalloc, cudaFree
 * or allocating routine.  With that workspace bf16 inputs at head dim 128 take
 * the single-pass tensor-core kernel and every other case the CUDA-core
 * kernel; the faster two-phase kernels need more workspace than any fixed
 * array could hold for long inputs.
 *
 * Arguments are those of gdn_prefill without the workspace, with fp32 states
 * and prepared inputs (no state_dtype, no input_form), plus
 *   device_status  optional device int32 (caller's memory, NULL to discard) that
 *                  receives this call's device-detected status (GDN_OK,
 *                  GDN_ERR_BAD_SEQLENS or GDN_ERR_DEVICE_TIMEOUT) in stream order.
 * Returns GDN_ERR_WORKSPACE if these sizes need more workspace than the 256-byte
 * built-in array; otherwise what gdn_prefill returns.
 *
 * The first call on each device resolves the array's device address
 * (cudaGetSymbolAddress) with that device current and keeps it for the life
 * of the process; make that first call before any stream capture.  A reset of
 * the device's primary context (cudaDeviceReset) invalidates that address: do
 * not call this entry point on a device after resetting it.  Every call on a
 * device shares the one array: each call clears its header first, and calls
 * whose work overlaps on the GPU (other streams, other host threads without
 * ordering) race on it.
 */
int32_t gdn_prefill_noalloc(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const int32_t *cu_seqlens, int32_t num_seqs,
                            int64_t total_tokens, int32_t num_qk_heads, int32_t num_v_heads,
                            int32_t head_dim_k, int32_t head_dim_v, int32_t dtype, int32_t o_dtype,
                            float scale, const float *initial_state, float *final_state, void *o,
                            int32_t *device_status, void *stream);

/*
 * Decode step: one new token for each of `batch` sequences, updating their
 * states in place ("Inside Qwen3.8-27B ...", section "Gated DeltaNet
 * Mechanics": in inference the state is updated token by token).
 *
 *   q, k     [batch, Hqk, Dk]        dtype
 *   v        [batch, Hv, Dv]         dtype
 *   g, beta  [batch, Hv]             fp32
 *   state    [batch, Hv, Dv, Dk]     fp32, read and overwritten in place
 *   o        [batch, Hv, Dv]         o_dtype (output); must not overlap state
 *
 * Supported: Hv % Hqk == 0; Dk, Dv in {64, 128}; dtype and o_dtype each bf16
 * or fp32.  Needs no workspace.  batch = 0 is a valid no-op.
 */
int32_t gdn_decode_step(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, float *state, void *o, int32_t batch,
                        int32_t num_qk_heads, int32_t num_v_heads, int32_t head_dim_k,
                        int32_t head_dim_v, int32_t dtype, int32_t o_dtype, float scale,
                        void *stream);

/*
 * Multi-token decode over a pool of states: `tokens` new tokens for each of
 * `batch` sequences, each sequence's state read from one slot of `state_in`
 * and written after the last token to one slot of `state_out`.  Serves
 * speculative verification (several drafted tokens per call, the state written
 * to a fresh slot so that a rejected draft leaves the old one intact) and
 * continuous batching (sequences bound to arbitrary slots, padding entries).
 * Same rule as gdn_decode_step, applied `tokens` times in order; each state is
 * read from HBM once and written once per call.  (The pages' inference mode
 * updates the state token by token: "Inside Qwen3.8-27B ...", section "Gated
 * DeltaNet Mechanics".)
 *
 *   q, k        [batch, tokens, Hqk, Dk]   dtype
 *   v           [batch, tokens, Hv, Dv]    dtype
 *   g, beta     [batch, tokens, Hv]        fp32
 *   state_in    [num_slots, Hv, Dv, Dk]    state_dtype, pool read
 *   state_out   [num_slots, Hv, Dv, Dk]    state_dtype, pool written; may be state_in
 *   src_slot    [batch] int32, device: slot of sequence b in state_in; NULL means
 *               slot b.  A negative entry marks padding: nothing is read or
 *               written for that sequence (its o is left untouched).
 *   dst_slot    [batch] int32, device: slot written in state_out; NULL means the
 *               source slot.  No two sequences may write the same slot, and a
 *               written slot must not be another sequence's source slot in the
 *               same call when state_out == state_in.
 *   o           [batch, tokens, Hv, Dv]    o_dtype (output)
 *   state_dtype GDN_DTYPE_FP32, or GDN_DTYPE_BF16 for states at rest in bf16
 *               (half the bytes per call).  The arithmetic is fp32 either way:
 *               a bf16 state is widened exactly on load, carried in fp32 through
 *               all `tokens` updates, and rounded to nearest even once, when it
 *               is stored.  The fixed state of all DeltaNet layers is put at
 *               some tens of megabytes in "Qwen3.8 Explained: 27B Multimodal,
 *               2.4T MoE, and the VRAM Math", section "The architecture detail
 *               that matters for VRAM"; bf16 at 48 layers x 48 heads x 128 x 128
 *               is 72 MiB.
 *   input_form  GDN_INPUT_PREPARED or GDN_INPUT_RAW (q, k normalised and g,
 *               beta mapped inside the kernel; see above).
 *   device_status  optional device int32 (caller's memory, NULL to discard): a
 *               slot index >= num_slots (or a negative dst_slot for a real
 *               sequence) is recorded as GDN_ERR_INVALID_ARG there (first error
 *               wins, as with the workspace status word) and that sequence is
 *               skipped.
 *
 * Supported: 1 <= tokens <= 16; Hv % Hqk == 0; Dk, Dv in {64, 128}; dtype and
 * o_dtype each bf16 or fp32.  batch = 0 or tokens = 0 is a valid no-op.
 */
int32_t gdn_decode_tokens(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const void *state_in, void *state_out,
                          const int32_t *src_slot, const int32_t *dst_slot, int32_t num_slots,
                          void *o, int32_t batch, int32_t tokens, int32_t num_qk_heads,
                          int32_t num_v_heads, int32_t head_dim_k, int32_t head_dim_v,
                          int32_t dtype, int32_t o_dtype, int32_t state_dtype,
                          int32_t input_form, float scale, int32_t *device_status, void *stream);

/*
 * Bytes of device workspace gdn_prefill_backward needs to run the chunk-form
 * backward (0 for invalid sizes): the status header and plan, then per
 * (64-token chunk, value head) the chunk's fp32 intermediates (Tm, P and
 * E . K K^T at 64 x 64; W, U~, U, dU, dW and two partial gradients at 64 x D;
 * the state and dL/dstate at the chunk's boundaries, Dv x Dk each; about
 * (T/64 + num_seqs) x Hv x (2 Dv Dk + 7 x 64 D + 3 x 64 x 64) x 4 bytes).  At
 * 8192 tokens, 48 value heads and D = 128 that is about 2.8 GB.  The value is at least the sequential size
 * below, so a workspace of this size always runs the chunk form.
 */
size_t gdn_prefill_backward_workspace_size(int32_t num_seqs, int64_t total_tokens,
                                           int32_t num_qk_heads, int32_t num_v_heads,
                                           int32_t head_dim_k, int32_t head_dim_v);

/*
 * Bytes of device workspace the sequential (token-by-token) backward needs
 * (0 for invalid sizes): the status header, a checkpoint of every state
 * every 16 tokens (about (T/16 + num_seqs) x Hv x Dv x Dk x 4 bytes), a
 * scratch of 16 states per (sequence, value head), and per-value-head dq, dk
 * when Hv > Hqk.  gdn_prefill_backward runs the sequential form when its
 * workspace holds at least this many bytes but fewer than
 * gdn_prefill_backward_workspace_size.
 */
size_t gdn_prefill_backward_workspace_size_sequential(int32_t num_seqs, int64_t total_tokens,
                                                      int32_t num_qk_heads, int32_t num_v_heads,
                                                      int32_t head_dim_k, int32_t head_dim_v);

/*
 * Backward pass of gdn_prefill (training): the gradients of a loss L with
 * respect to q, k, v, g, beta and the initial state, given d_o = dL/do and
 * optionally d_final_state = dL/dS_final.  Same rule, layout and sequences as
 * gdn_prefill with fp32 states and prepared inputs (the page's note says the
 * block form is used in training as well: "Inside Qwen3.8-27B ...", section
 * "Gated DeltaNet Mechanics").
 *
 * Two algorithms, chosen by the workspace size, both fp32-accurate:
 *   - chunk form (workspace >= gdn_prefill_backward_workspace_size): the
 *     reverse mode of the chunked WY/UT form.  Per 64-token chunk with
 *     E_ts = e^{G_t - G_s}, P = E . Q K^T, Tm = (I + A)^-1 and
 *     U = U~ - W S0^T as in gdn_prefill, going backwards over the chunks
 *     with dO' = scale d_o and dS1 = dL/d(state after the chunk):
 *       dU = P^T dO' + diag(kdec) K dS1^T;
 *       dS0 = gamma_C dS1 + dO'^T diag(gamma) Q - dU^T W;
 *     then every chunk on its own: dQ, dK, dV, dbeta and dG through the
 *     products of the WY/UT transform (dA = -Tm^T dT Tm^T) and dg as suffix
 *     sums of dG within the chunk.  The dense products run on tensor cores
 *     at about fp32 accuracy: fp32 operands split into hi and lo parts and
 *     three products (hi*hi + hi*lo + lo*hi), raw bf16 inputs used as they
 *     are; the products with the chunk states on tcgen05, the rest as
 *     warp-level MMAs.  g is clamped at -30 as in the tensor-core prefill.
 *     The forward and reverse chains run in one launch; the call is
 *     stream-ordered on `stream` (it can be captured in a CUDA graph).
 *   - sequential (at least gdn_prefill_backward_workspace_size_sequential
 *     bytes): the token-by-token rule on CUDA cores.  With u = S_{t-1} k_t,
 *     w = v_t - alpha_t u and G = dL/dS_t, going backwards over the tokens:
 *       G += scale dO_t q_t^T;  dq_t = scale S_t^T dO_t;  dv_t = beta_t G k_t;
 *       dbeta_t = w . G k_t;  dg_t = alpha_t (<G, S_{t-1}> - beta_t (G k_t) . u);
 *       dk_t = beta_t G^T w - alpha_t beta_t S_{t-1}^T G k_t;
 *       G <- alpha_t (G - beta_t (G k_t) k_t^T);  d_initial_state = G at the start.
 * dq and dk of a query/key head sum over the value heads reading it, in a
 * fixed order (results do not depend on scheduling).
 *
 *   q, k, v, g, beta, cu_seqlens, initial_state (fp32 or NULL), scale: as for
 *                  gdn_prefill (prepared inputs; dtype bf16 or fp32)
 *   d_o            [T, Hv, Dv] fp32
 *   d_final_state  [num_seqs, Hv, Dv, Dk] fp32, or NULL for zeros
 *   dq, dk         [T, Hqk, Dk] fp32 (outputs);  dv [T, Hv, Dv] fp32;
 *   dg, dbeta      [T, Hv] fp32;  d_initial_state [num_seqs, Hv, Dv, Dk] fp32 or NULL
 *   workspace      256-byte aligned, sized as above; its first word is the
 *                  sticky device status word (GDN_ERR_BAD_SEQLENS), read with
 *                  gdn_get_device_status.  Smaller than the sequential size:
 *                  GDN_ERR_WORKSPACE.
 * Supported: Hv % Hqk == 0; Dk, Dv in {64, 128}.
 */
int32_t gdn_prefill_backward(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const int32_t *cu_seqlens, int32_t num_seqs,
                             int64_t total_tokens, int32_t num_qk_heads, int32_t num_v_heads,
                             int32_t head_dim_k, int32_t head_dim_v, int32_t dtype, float scale,
                             const float *initial_state, const float *d_o,
                             const float *d_final_state, float *dq, float *dk, float *dv,
                             float *dg, float *dbeta, float *d_initial_state, void *workspace,
                             size_t workspace_bytes, void *stream);

/*
 * The sequential backward on its own, whatever the workspace size: same
 * arguments and results as gdn_prefill_backward; the workspace must hold at
 * least gdn_prefill_backward_workspace_size_sequential bytes.
 */
int32_t gdn_prefill_backward_sequential(const void *q, const void *k, const void *v, const float *g,
                                        const float *beta, const int32_t *cu_seqlens,
                                        int32_t num_seqs, int64_t total_tokens,
                                        int32_t num_qk_heads, int32_t num_v_heads,
                                        int32_t head_dim_k, int32_t head_dim_v, int32_t dtype,
                                        float scale, const float *initial_state, const float *d_o,
                                        const float *d_final_state, float *dq, float *dk,
                                        float *dv, float *dg, float *dbeta, float *d_initial_state,
                                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * 1 if gdn_prefill with these sizes and dtype runs the tensor-core (tcgen05)
 * kernel, 0 if it runs the fp32 CUDA-core kernel or the arguments are invalid.
 * Host only; touches no device.
 */
int32_t gdn_prefill_uses_tensor_cores(int32_t num_qk_heads, int32_t num_v_heads,
                                      int32_t head_dim_k, int32_t head_dim_v, int32_t dtype);

/*
 * Synchronise `stream`, read the status word kept in `workspace` (the first
 * device-detected error of the gdn_prefill calls that used it since it was
 * last cleared, or GDN_OK), store it in *status_host (host pointer) and clear
 * it.  Returns GDN_OK when the read itself worked.
 */
int32_t gdn_get_device_status(const void *workspace, void *stream, int32_t *status_host);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
