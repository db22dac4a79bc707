/*
 * gdn.h -- C ABI of libgdn.so, a B200 (sm_100a) implementation of the Gated
 * DeltaNet (GDN) token mixer.
 *
 * The operations follow "On the design of Qwen3.8-Next architecture: evaluation,
 * efficiency and training stability" (paper-archivist reading of arXiv
 * 2608.30320), section 2.1.1:
 *   "Gated Delta recurrence", eqs. (1)-(5):
 *       S~_{t-1} = alpha_t S_{t-1}                  (1)
 *       e_t      = v_t - S~_{t-1}^T k_t             (2)
 *       S_t      = S~_{t-1} + beta_t k_t e_t^T      (3)
 *       y_t      = S_t^T q_t                        (4)
 *     with S_t in R^{dk x dv} (the transpose of the original GDN convention).
 *   "GDN parameterisation", eqs. (6)-(11): ShortConv -> SiLU -> L2Norm for q and
 *     k, ShortConv -> SiLU for v, beta = sigmoid(.), alpha = exp(-exp(A)
 *     softplus(. + b)), and the sigmoid output gate over a zero-centred RMSNorm.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout.   Token-major, head-minor: q, k are [N, H, dk], v, y, z are [N, H, dv],
 *           per-token scalars (g, beta, logits) are [N, H]; the innermost index
 *           is contiguous.  A state is [rows, H, dk, dv] fp32, dv contiguous.
 *           N counts all tokens of all packed sequences.
 * Sequences. cu_seqlens (int32, [num_seqs+1], cu[0] = 0, non-decreasing,
 *           cu[num_seqs] <= N) gives packed variable-length sequences; NULL means
 *           num_seqs sequences of N/num_seqs tokens each.  Every sequence starts
 *           from its own initial state row and a zero convolution history.
 * Decay.    alpha is passed as g = log(alpha) (fp32): the chunked algorithm works
 *           with cumulative log-decays, and alpha itself can underflow in fp32.
 * Memory.   Every pointer is a DEVICE pointer owned by the caller, 16-byte
 *           aligned.  The compute calls allocate nothing and keep no per-call state
 *           (gdn_chunk_fwd_noalloc's scratch is part of the library's device image;
 *           only the timing calls create CUDA events); calls are re-entrant from
 *           several host threads.
 * Streams.  `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *           only enqueues work on it and returns; nothing synchronises.
 * Errors.   Argument errors are detected on the host before anything is enqueued
 *           and return GDN_ERR_INVALID_ARG (bad value) or GDN_ERR_UNSUPPORTED
 *           (valid but not implemented).  A failed launch returns GDN_ERR_CUDA.
 *           Device-side bounded waits that run out record a code in a device error
 *           word, read by gdn_check_device_error.  gdn_last_error_message gives a
 *           one-line reason for the calling thread's last failure.  No C++
 *           exception crosses this interface.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* gdn_stream_t; /* a cudaStream_t */

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,
    GDN_ERR_UNSUPPORTED = 2,
    GDN_ERR_CUDA = 3,
    GDN_ERR_TIMEOUT = 4
} gdn_status_t;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1, GDN_F16 = 2 } gdn_dtype_t;

/* Library version, major*10000 + minor*100 + patch. */
int gdn_version(void);

/* 1 for the bounds-checking build (libgdn_debug.so, compiled with -DGDN_BOUNDS_CHECK), else 0.
 * In that build the kernels test their computed global indices (state blocks of decode slots,
 * chunk records and token rows, checkpoint blocks, output rows) against the tensors' extents
 * that the call's sizes imply; an index outside them is not accessed, and
 * gdn_check_device_error then returns GDN_ERR_INVALID_ARG naming the bounds check.  Results of
 * a call that trips no check are those of the release build. */
int gdn_bounds_checked(void);

/* Static string naming a status code. */
const char* gdn_status_string(gdn_status_t status);

/* One-line reason for the calling thread's most recent non-OK return ("" if none). */
const char* gdn_last_error_message(void);

/*
 * Synchronises `stream`, then reads and clears the current device's error word.
 * Returns GDN_ERR_TIMEOUT if a kernel's bounded wait ran out since the last check,
 * GDN_ERR_INVALID_ARG if a kernel found cu_seqlens out of order / range or a state
 * slot out of range, GDN_ERR_CUDA if the stream reports a CUDA error, else GDN_OK.
 */
gdn_status_t gdn_check_device_error(gdn_stream_t stream);

/*
 * Test knob: the clock64 budget of every device-side wait (0 restores the default
 * of about one second).  Process-wide; affects kernels launched after the call.
 */
void gdn_set_wait_budget(uint64_t cycles);

/*
 * Per-kernel launch timing (a measurement aid; the pages define no such call).
 * gdn_timing_start: from now on every kernel launch of the library on the current
 *   device is bracketed by two CUDA events recorded on the launch's stream, for at most
 *   max_launches launches (later ones run untimed).  The event pool (2 * max_launches
 *   events) is created here.  GDN_ERR_INVALID_ARG if timing is already on or
 *   max_launches is outside [1, 2^20]; GDN_ERR_CUDA if the events cannot be created.
 *   Do not start timing while a stream is being captured into a CUDA graph.
 * gdn_timing_stop: waits for the recorded events, aggregates them per kernel name in
 *   order of first launch, and turns timing off.  Up to cap entries are written:
 *   names[i] (a static string owned by the library), launches[i], total_ms[i] (sum of
 *   the launches' device durations).  *n_kernels (nullable) receives the number of
 *   distinct kernels, which may exceed cap.  GDN_ERR_INVALID_ARG if timing is off.
 */
gdn_status_t gdn_timing_start(int max_launches);
gdn_status_t gdn_timing_stop(int cap, const char** names, int* launches, double* total_ms,
                             int* n_kernels);

/*
 * gdn_prep -- eqs. (6)-(10): the input side of the mixer.
 *   q = L2Norm(SiLU(ShortConv(x_q)))   (6)     k = L2Norm(SiLU(ShortConv(x_k)))   (7)
 *   v = SiLU(ShortConv(x_v))           (8)     beta = sigmoid(beta_logit)         (9)
 *   g = log alpha = -exp(A_log[h]) * softplus(alpha_logit + alpha_bias[h])         (10)
 * ShortConv is causal and depthwise with conv_width taps and no bias:
 *   conv[t, c] = sum_{j<W} w[c][j] * x[t-(W-1)+j, c], zero before the sequence start,
 * with channel c = h*d + i and w stored [H*d, W] fp32 (tap W-1 meets token t).
 * L2Norm(x) = x / sqrt(sum_i x_i^2 + l2_eps) over the head dimension.
 *   x_q, x_k [N,H,dk], x_v [N,H,dv], beta_logit, alpha_logit [N,H]: in_dtype.
 *   A_log, alpha_bias [H] fp32.   q, k [N,H,dk], v [N,H,dv]: out_dtype.
 *   g_out, beta_out [N,H] fp32.   conv_width in [1, 8].  dk, dv in {16,32,64,128}.
 * Tokens at index >= cu_seqlens[num_seqs] are left untouched.
 */
gdn_status_t gdn_prep(const void* x_q, const void* x_k, const void* x_v, const float* conv_w_q,
                      const float* conv_w_k, const float* conv_w_v, int conv_width,
                      const void* beta_logit, const void* alpha_logit, const float* A_log,
                      const float* alpha_bias, const int32_t* cu_seqlens, int num_seqs, int N, int H,
                      int dk, int dv, float l2_eps, gdn_dtype_t in_dtype, gdn_dtype_t out_dtype,
                      void* q, void* k, void* v, float* g_out, float* beta_out, gdn_stream_t stream);

/*
 * gdn_inproj_prep -- the mixer's input projections fused with eqs. (6)-(10): from the
 * normalised residual stream x_t (section 2.1.1, "GDN parameterisation") the six products
 * W_q x_t, W_k x_t, W_v x_t, W_z x_t, W_beta x_t, W_alpha x_t as one tensor-core matrix
 * product, then, on its fp32 results, exactly gdn_prep's steps (ShortConv -> SiLU -> L2Norm
 * for q and k, ShortConv -> SiLU for v, eqs. (9)-(10) for beta and g).  The raw projections
 * are never stored; z = W_z x_t (the input of eq. (11)'s gate) is stored as is.
 *   x [N, D] in_dtype (BF16 or F16), row-major; D a multiple of 64.
 *   w [4*H*d + 2*H, D] in_dtype: the rows (out_features x in_features) of W_q, W_k, W_v, W_z
 *     (H*d rows each, row h*d + i is channel i of head h), then W_beta and W_alpha (H rows each).
 *   conv_w_*, conv_width, A_log, alpha_bias, cu_seqlens, num_seqs, l2_eps as in gdn_prep.
 *   q, k, v [N,H,d] and z [N,H,d] (NULL: W_z is not applied): out_dtype (BF16 or F16).
 *   g_out, beta_out [N,H] fp32.
 * Built for dk = dv = d = 128 and H a multiple of 16 up to 128 (others: GDN_ERR_UNSUPPORTED).
 * q, k, v of tokens at index >= cu_seqlens[num_seqs] are left untouched; z, g and beta are
 * written for all N tokens.  Nothing is allocated; asynchronous on the stream.
 */
gdn_status_t gdn_inproj_prep(const void* x, const void* w, int D, const float* conv_w_q,
                             const float* conv_w_k, const float* conv_w_v, int conv_width,
                             const float* A_log, const float* alpha_bias, const int32_t* cu_seqlens,
                             int num_seqs, int N, int H, int dk, int dv, float l2_eps,
                             gdn_dtype_t in_dtype, gdn_dtype_t out_dtype, void* q, void* k, void* v,
                             void* z, float* g_out, float* beta_out, gdn_stream_t stream);

/*
 * gdn_chunk_fwd -- prefill: eqs. (1)-(4) over every token of every packed sequence.
 *   q, k [N,H,dk], v [N,H,dv]: in_dtype.  g = log alpha, beta [N,H]: fp32.
 *   S0 [num_seqs,H,dk,dv] fp32 or NULL (zero initial state).
 *   y [N,H,dv]: y_dtype.  S_T [num_seqs,H,dk,dv] fp32 (final state) or NULL.
 *   scale multiplies the readout (y_t = scale * S_t^T q_t); 1.0 is eq. (4) as printed.
 * chunk selects the algorithm:
 *   chunk = 0: token-sequential fp32 recurrence on CUDA cores (any supported
 *              shape and dtype; exact up to fp32 rounding order).
 *   chunk = 64: chunkwise-parallel form on the tensor cores
 *              (requires dk = dv = 128 and in_dtype BF16 or F16; other shapes and
 *              chunk sizes return GDN_ERR_UNSUPPORTED).  It is derived
 *              from eq. (5): within a chunk, the UT transform T = (I + A)^-1 with
 *              A[r,s] = beta_r exp(gamma_r - gamma_s) k_r.k_s turns the token loop
 *              into dense products (one kernel per (chunk, head), warp-level mma);
 *              between chunks a second kernel carries the fp32 state through tcgen05
 *              products with TMEM accumulators.
 * workspace: device scratch of at least gdn_chunk_fwd_workspace_size(...) bytes
 * (may be NULL when that size is 0).  Tokens at index >= cu_seqlens[num_seqs] are
 * neither read nor written.  N = 0 (every sequence empty): nothing is done without S_T;
 * with S_T, it receives S0 (zeros when S0 is NULL), and q, k, v, g, beta, y and the
 * workspace may be NULL.
 */
size_t gdn_chunk_fwd_workspace_size(int N, int num_seqs, int H, int dk, int dv, int chunk);

gdn_status_t gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, const float* S0, const int32_t* cu_seqlens,
                           int num_seqs, int N, int H, int dk, int dv, int chunk, float scale,
                           gdn_dtype_t in_dtype, gdn_dtype_t y_dtype, void* y, float* S_T,
                           void* workspace, size_t workspace_bytes, gdn_stream_t stream);

/*
 * gdn_chunk_fwd_gated -- gdn_chunk_fwd (chunk = 64) with eq. (11)'s output gate, without
 * the projection W_o, fused into the chunked pass, so y never goes to memory:
 *   out[t,h,:] = sigmoid(z[t,h,:]) * y[t,h,:] / sqrt(mean_i y[t,h,i]^2 + eps) * (1 + norm_w)
 * Arguments as gdn_chunk_fwd, except: no y / y_dtype; z and out [N,H,dv] in io_dtype
 * (BF16 or F16); norm_w [dv] fp32, shared by all heads; eps >= 0.  Tensor-core path only:
 * chunk = 64, dk = dv = 128, in_dtype BF16 or F16 (anything else returns
 * GDN_ERR_UNSUPPORTED; use gdn_chunk_fwd followed by gdn_out_gate).  The four 32-column dv slabs of a (sequence,
 * head) run as one thread-block cluster and exchange each row's partial sum of squares
 * through distributed shared memory.  Same workspace as gdn_chunk_fwd.
 */
gdn_status_t gdn_chunk_fwd_gated(const void* q, const void* k, const void* v, const float* g,
                                 const float* beta, const float* S0, const int32_t* cu_seqlens,
                                 int num_seqs, int N, int H, int dk, int dv, int chunk, float scale,
                                 gdn_dtype_t in_dtype, const void* z, const float* norm_w, float eps,
                                 gdn_dtype_t io_dtype, void* out, float* S_T, void* workspace,
                                 size_t workspace_bytes, gdn_stream_t stream);

/*
 * gdn_chunk_fwd_noalloc -- gdn_chunk_fwd for callers that cannot allocate device memory.
 * (An addition of this library; the paper has no counterpart.)
 *
 * Some callers cannot obtain scratch memory at call time: a serving loop whose device
 * memory is fixed at start-up, a plugin whose host process owns every device
 * allocation, or code on a path where cudaMalloc's implicit device synchronisation is
 * not acceptable.  This entry point takes the same arguments as gdn_chunk_fwd minus the
 * workspace, and uses instead a scratch array of GDN_NOALLOC_SCRATCH_BYTES (64 MiB)
 * that is part of the library's device image: every GPU that loads the library holds
 * it until the process exits.  It calls no cudaMalloc, cudaFree or allocating library
 * routine.
 *   - A call whose scratch need, gdn_chunk_fwd_workspace_size(N, num_seqs, H, dk, dv,
 *     chunk), exceeds GDN_NOALLOC_SCRATCH_BYTES returns GDN_ERR_INVALID_ARG with the
 *     two sizes in gdn_last_error_message().  (chunk = 0 needs no scratch.)
 *   - The first call in a CUDA context (the device's primary context, or whichever
 *     context is current on the calling thread) looks up that context's address of the
 *     array (cudaGetSymbolAddress); make that first call before any stream capture.
 *     Later calls in the same context reuse the address; after the context is destroyed
 *     (e.g. cudaDeviceReset) the next call looks it up again.
 *   - Arguments the tensor-core path does not accept (other chunk sizes, head sizes or an
 *     fp32 input) need no scratch and get gdn_chunk_fwd's own answer.
 *   - All calls share the one array, which keeps the last call's contents; every
 *     record a call reads was written earlier in the same call, so nothing needs
 *     clearing.  Calls that overlap on the GPU (different streams, or devices sharing
 *     a context) race on the array and give undefined results: serialise them.
 */
#define GDN_NOALLOC_SCRATCH_BYTES (64ull << 20)

gdn_status_t gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* g,
                                   const float* beta, const float* S0, const int32_t* cu_seqlens,
                                   int num_seqs, int N, int H, int dk, int dv, int chunk,
                                   float scale, gdn_dtype_t in_dtype, gdn_dtype_t y_dtype,
                                   void* y, float* S_T, gdn_stream_t stream);

/*
 * gdn_chunk_fwd_prep -- gdn_prep (eqs. (6)-(10)) fused into gdn_chunk_fwd's chunked pass: the
 * projection outputs x_q, x_k, x_v go through ShortConv -> SiLU (-> L2Norm) inside the chunk
 * kernel, and q, k, v, g, beta are never stored as tensors (the per-chunk records carry what the
 * sequential pass needs).  Arguments as gdn_prep and gdn_chunk_fwd:
 *   x_q, x_k, x_v [N,H,128], beta_logit, alpha_logit [N,H]: in_dtype (BF16 or F16).
 *   conv_w_* [H*128, conv_width] fp32, conv_width in [1, 8]; A_log, alpha_bias [H] fp32.
 *   qkv_dtype (BF16 or F16): the format q, k, v are rounded to before eqs. (1)-(4), as
 *   gdn_prep's out_dtype would store them; the products then run on it.
 *   S0, cu_seqlens, y, S_T, scale as in gdn_chunk_fwd.
 * Only chunk = 64 and dk = dv = 128 are built (others: GDN_ERR_UNSUPPORTED).
 * workspace: at least gdn_chunk_fwd_prep_workspace_size(...) bytes.
 */
size_t gdn_chunk_fwd_prep_workspace_size(int N, int num_seqs, int H, int dk, int dv, int chunk);

gdn_status_t gdn_chunk_fwd_prep(const void* x_q, const void* x_k, const void* x_v, const float* conv_w_q,
                                const float* conv_w_k, const float* conv_w_v, int conv_width,
                                const void* beta_logit, const void* alpha_logit, const float* A_log,
                                const float* alpha_bias, float l2_eps, const float* S0,
                                const int32_t* cu_seqlens, int num_seqs, int N, int H, int dk, int dv,
                                int chunk, float scale, gdn_dtype_t in_dtype, gdn_dtype_t qkv_dtype,
                                gdn_dtype_t y_dtype, void* y, float* S_T, void* workspace,
                                size_t workspace_bytes, gdn_stream_t stream);

/*
 * gdn_chunk_bwd -- gradients through eqs. (1)-(4) for packed sequences (the backward of
 * gdn_chunk_fwd): for a loss L with dL/dy = dy and dL/dS_T = dS_T (NULL: zero), returns dL/dq,
 * dL/dk, dL/dv, dL/dg (g = log alpha), dL/dbeta and dL/dS0.  Each token step
 *   S~ = alpha S, e = v - S~^T k, S_t = S~ + beta k e^T, y = scale S_t^T q
 * is walked backwards with D = dL/dS_t:
 *   D += scale q dy^T; dq = scale S_t dy; de = beta D^T k; dbeta = k^T D e;
 *   dk = beta D e - S~ de; dv = de; D~ = D - k de^T; dg = alpha <D~, S>; D <- alpha D~.
 * The states come from a forward pass that checkpoints every 8 tokens into the workspace.
 *   q, k, v, g, beta, S0, cu_seqlens, scale, in_dtype as given to gdn_chunk_fwd; dy [N,H,dv]
 *   in dy_dtype; dS_T [num_seqs,H,dk,dv] fp32 or NULL.  Outputs, fp32: dq, dk [N,H,dk],
 *   dv [N,H,dv], dg, dbeta [N,H], dS0 [num_seqs,H,dk,dv].  dq, dk, dg, dbeta are zeroed for
 *   all N tokens and accumulated over 32-column slabs of the state with atomic adds, so their
 *   last bits depend on the order of those adds; dv of tokens in no sequence is not written.
 * workspace: at least gdn_chunk_bwd_workspace_size(...) bytes (the checkpoints).
 */
size_t gdn_chunk_bwd_workspace_size(int N, int num_seqs, int H, int dk, int dv);

gdn_status_t gdn_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                           const float* S0, const int32_t* cu_seqlens, int num_seqs, int N, int H, int dk,
                           int dv, float scale, gdn_dtype_t in_dtype, const void* dy, gdn_dtype_t dy_dtype,
                           const float* dS_T, float* dq, float* dk_out, float* dv_out, float* dg,
                           float* dbeta, float* dS0, void* workspace, size_t workspace_bytes,
                           gdn_stream_t stream);

/*
 * gdn_decode_step -- one token per row against a resident state, eqs. (1)-(4):
 *   S <- alpha S + beta k e^T with e = v - alpha S^T k, y = scale * S^T q (new S).
 *   q, k [B,H,dk], v [B,H,dv]: in_dtype.  g, beta [B,H] fp32.
 *   state [num_slots,H,dk,dv] fp32, read and written in place; row b uses
 *   state[state_slot[b]] (int32 [B], NULL = row b uses slot b, which needs
 *   num_slots >= B).  Two rows must not name the same slot.  A row whose slot is
 *   outside [0, num_slots) is skipped and flagged in the device error word
 *   (gdn_check_device_error then returns GDN_ERR_INVALID_ARG).  y [B,H,dv]: y_dtype.
 */
gdn_status_t gdn_decode_step(const void* q, const void* k, const void* v, const float* g,
                             const float* beta, float* state, const int32_t* state_slot,
                             int num_slots, int B, int H, int dk, int dv, float scale,
                             gdn_dtype_t in_dtype,
                             gdn_dtype_t y_dtype, void* y, gdn_stream_t stream);

/*
 * gdn_mixer_decode_step -- one token per row through the whole mixer of section 2.1.1, one
 * kernel: eqs. (6)-(10) on the token's projection outputs and the row's causal conv history,
 * eqs. (1)-(4) against the resident state, and eq. (11)'s output gate (without W_o).  q, k, v
 * stay in fp32 inside the kernel (never stored).
 *   x_q, x_k [B,H,dk], x_v [B,H,dv], beta_logit, alpha_logit [B,H], z [B,H,dv]: in_dtype.
 *   conv_w_q, conv_w_k [H*dk, W], conv_w_v [H*dv, W] fp32 (W = conv_width in [1, 8]; tap W-1
 *     meets the current token, as in gdn_prep); A_log, alpha_bias [H] fp32; norm_w [dv] fp32.
 *   conv_state [num_slots, W-1, H, 2*dk + dv] in_dtype: for each slot the W-1 previous raw
 *     inputs, oldest first, each one head's q channels, then k, then v.  Read and shifted in
 *     place: afterwards it holds the W-1 newest inputs, the current one last.  A new sequence
 *     starts from zeros (the zero history of a sequence start).  May be NULL when W = 1.
 *   state [num_slots,H,dk,dv] fp32, in place; state_slot as in gdn_decode_step (row b uses slot
 *     state_slot[b] of both state and conv_state).
 *   out [B,H,dv]: out_dtype.  l2_eps inside the L2Norm square root, rms_eps inside the RMSNorm
 *   one; scale multiplies the readout as in gdn_chunk_fwd.
 */
gdn_status_t gdn_mixer_decode_step(const void* x_q, const void* x_k, const void* x_v, const float* conv_w_q,
                                   const float* conv_w_k, const float* conv_w_v, int conv_width,
                                   const void* beta_logit, const void* alpha_logit, const float* A_log,
                                   const float* alpha_bias, const void* z, const float* norm_w, float l2_eps,
                                   float rms_eps, void* conv_state, float* state, const int32_t* state_slot,
                                   int num_slots, int B, int H, int dk, int dv, float scale, gdn_dtype_t in_dtype,
                                   gdn_dtype_t out_dtype, void* out, gdn_stream_t stream);

/*
 * gdn_out_gate -- eq. (11) without the output projection W_o:
 *   out = sigmoid(z) * y / sqrt(mean_dv(y^2) + eps) * (1 + norm_w)
 * per (token, head) over dv; norm_w [dv] fp32 is shared by all heads (the
 * zero-centred RMSNorm weight).  y [N,H,dv]: y_dtype; z, out [N,H,dv]: io_dtype.
 */
gdn_status_t gdn_out_gate(const void* y, const void* z, const float* norm_w, float eps, int N, int H,
                          int dv, gdn_dtype_t y_dtype, gdn_dtype_t io_dtype, void* out,
                          gdn_stream_t stream);

/*
 * gdn_state_map_apply -- S_out = M S_in + B for each of `rows` states: a sequence segment's
 * affine map applied to a state, the step that gives a rank of a context-parallel prefill its
 * initial state.  Eq. (5) (S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T) is
 * affine in S_{t-1}, so a segment maps S_start to M S_start + B, where M [dk,dk] is the
 * segment's state after starting from S = I with v = 0 and B [dk,dv] its state after starting
 * from S = 0 (both are S_T outputs of gdn_chunk_fwd).
 *   M [rows,dk,dk], B [rows,dk,dv] (NULL: zero), S_in, S_out [rows,dk,dv]: fp32, row-major.
 *   S_out must not overlap M, B or S_in.  dk, dv in {16,32,64,128}.  fp32 accumulation.
 */
gdn_status_t gdn_state_map_apply(const float* M, const float* B, const float* S_in, float* S_out, int rows,
                                 int dk, int dv, gdn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
