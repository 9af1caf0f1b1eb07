/*
 * gdn.h -- C ABI of the B200 (sm_100a) gated delta rule library, libgdn_b200.so.
 *
 * The library computes the Gated DeltaNet token mixer's gated delta rule (chunked prefill,
 * one- and several-token decode, and the gradients), its output epilogue and the feature
 * and gate step in front of it, as defined on the joezjh.github.io notes page "Qwen3.8-Flash-Next"
 * (section "Gated DeltaNet 核心机制", the four-line update rule and its equivalent
 * form; section "GDN 参数化细节", the output-gate equation) and on the pwwt.cn
 * translation of the report (section 2.1.1, "sigmoid output gate", "zero-centred
 * RMSNorm"). Per head, with state S in R^{d_k x d_v}:
 *
 *     S~ = alpha_t S_{t-1};  e_t = v_t - S~^T k_t;  S_t = S~ + beta_t k_t e_t^T;
 *     y_t = S_t^T (scale * q_t)            (equivalently S_t = alpha_t (I - beta_t k_t k_t^T)
 *                                            S_{t-1} + beta_t k_t v_t^T)
 *     o_t = sigmoid(z_t) * y_t / sqrt(mean(y_t^2) + eps) * (1 + w)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor argument is a DEVICE pointer owned by the caller (cudaMalloc'd or a
 *    torch tensor's data pointer), contiguous, in the layout stated. Pointers to q, k,
 *    v, y, z, o, S0, S_T and S must be 16-byte aligned; log_alpha/alpha/beta and
 *    cu_seqlens_dev 4-byte aligned.
 *  - STATE LAYOUT is value-major: [.., d_v, d_k], i.e. the transpose S^T stored
 *    row-major with the key dimension contiguous. (Row j holds column j of the pages'
 *    S.) All states in and out are fp32.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = the
 *    legacy default stream) and never synchronise, except gdn_device_error().
 *  - The library allocates no device memory in any call.
 *  - Outputs must not alias inputs, except S in gdn_decode_step, which is updated in
 *    place.
 *  - Argument errors are reported before any launch: GDN_ERR_INVALID_ARG (null or
 *    misaligned pointer, negative size, inconsistent cu_seqlens) or
 *    GDN_ERR_UNSUPPORTED (a size outside the supported set). A failed launch returns
 *    GDN_ERR_CUDA. Conditions a kernel detects while running (a bounded wait that
 *    gave up, an internal check) set a device-side error word that gdn_device_error()
 *    reads. No exception or abort crosses this boundary.
 *  - Not thread-safe with respect to gdn_device_error(): the error word is per device.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, bad cu_seqlens      */
    GDN_ERR_UNSUPPORTED = 2,   /* valid but outside the supported shapes/dtypes          */
    GDN_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed                   */
    GDN_ERR_TIMEOUT = 4,       /* (device error word) a bounded wait inside a kernel     */
    GDN_ERR_DEVICE_CHECK = 5   /* (device error word) an in-kernel consistency check     */
} gdn_status;

typedef enum {
    GDN_F32 = 0,               /* IEEE binary32                                          */
    GDN_BF16 = 1               /* bfloat16; results rounded to nearest even              */
} gdn_dtype;

/*
 * gdn_chunk_fwd -- chunked prefill of the gated delta rule over packed sequences.
 *
 * Defines: the four-line update rule above, applied token by token within each
 * sequence (joezjh.github.io notes, "Gated DeltaNet 核心机制"); the library computes it
 * in the chunkwise-parallel form (exact up to rounding), chunk tokens at a time.
 * Sequences are independent; the state starts at S0 (or 0) at each sequence start.
 *
 *   q, k        [N_tok, H, d_k]  in in_dtype (N_tok = cu_seqlens[n_seq]); the
 *                                parameterisation expects L2-normalised q, k
 *   v           [N_tok, H, d_v]  in in_dtype
 *   log_alpha   [N_tok, H] fp32  log of the decay gate, <= 0 (alpha in (0, 1])
 *   beta        [N_tok, H] fp32  write strength, in [0, 1]
 *   S0          [n_seq, H, d_v, d_k] fp32, or NULL for a zero initial state
 *   cu_seqlens_dev  [n_seq + 1] int32, device copy read by the kernels
 *   cu_seqlens_host [n_seq + 1] int32, HOST copy with identical contents, used to
 *                   validate and size the launch without a device->host copy;
 *                   element 0 must be 0 and the sequence non-decreasing
 *   n_seq >= 0, H >= 1
 *   d_k, d_v    each in {16, 32, 64, 128}
 *   chunk       in {16, 32, 64}; chunk boundaries restart at every sequence start
 *   scale       multiplies q (the pages use none: pass 1.0)
 *   y           [N_tok, H, d_v]  out, in y_dtype (GDN_F32 or GDN_BF16, independent of
 *               in_dtype; a bf16 y is the round-to-nearest-even of the fp32 result)
 *   S_T         [n_seq, H, d_v, d_k] fp32 out (final state per sequence), or NULL
 *   workspace   device scratch of workspace_bytes >= gdn_chunk_fwd_workspace_bytes(..),
 *               128-byte aligned (may be NULL when that is 0). The tensor-core path uses
 *               it as a ring of fp16 K tiles per SM id (64 KB for each id the device's
 *               SMs can report, %nsmid, at least the SM count); no initial contents are
 *               needed and nothing is left in it. Calls on different streams may share one
 *               workspace (each SM id's region is used by at most one cluster at a time).
 *               Caller-owned. An SM id beyond the workspace's regions is recorded as
 *               GDN_ERR_DEVICE_CHECK (gdn_device_error) and that chain is not computed.
 *
 * Paths: bf16 inputs with d_k = d_v = 128 and chunk = 64 run the sm_100a tensor-core
 * kernel (tcgen05 MMA with TMEM accumulators, TMA loads, fp32 state carry; bf16 inputs
 * feed the K K^T / Q K^T product, all other products use fp16 operands -- the inputs
 * convert exactly -- which requires the scaled q, k, v, S0, the state and the derived
 * operands to stay below 65520 in magnitude; the kernel checks every value it converts and
 * records GDN_ERR_DEVICE_CHECK (gdn_device_error) when one does not, or is NaN: the
 * outputs of that call are then unspecified); every other supported case runs the
 * CUDA-core fp32 chunk kernel.
 */
/* Scratch bytes gdn_chunk_fwd needs for these sizes on the current device: 64 KB per SM
 * id when d_k = d_v = 128 and chunk = 64 (the tensor-core path; sized for any input
 * dtype), else 0. Returns 0 when no device can be queried. The first call on a device reads
 * its SM id range with a one-thread kernel and a synchronous copy (once per device and
 * process): make it before any stream capture. */
size_t gdn_chunk_fwd_workspace_bytes(int n_seq, int64_t total_tokens, int H, int d_k, int d_v,
                                     int chunk);

gdn_status gdn_chunk_fwd(const void *q, const void *k, const void *v, gdn_dtype in_dtype,
                         const float *log_alpha, const float *beta, const float *S0,
                         const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                         int n_seq, int H, int d_k, int d_v, int chunk, float scale,
                         void *y, gdn_dtype y_dtype, float *S_T, void *workspace,
                         size_t workspace_bytes, void *stream);

/*
 * gdn_chunk_fwd_noalloc -- gdn_chunk_fwd without a caller workspace, for callers that
 * may not allocate (no counterpart in the pages: a deployment convenience, not part of
 * the method).
 *
 * Same arguments, results and errors as gdn_chunk_fwd, minus workspace. The scratch of
 * the tensor-core path is a fixed file-scope device array of the library (one per
 * device, 160 SM ids x 64 KB = 10 MB, reached through cudaGetSymbolAddress); the call
 * allocates and frees nothing. A device whose SM ids (%nsmid) exceed 160 returns
 * GDN_ERR_UNSUPPORTED. The first call on a device reads that range once (a one-thread
 * kernel and a synchronous copy): make it before any stream capture. The array is shared by every call in the process: overlapping
 * calls on different streams do not race only because each SM id's region is used by at
 * most one cluster at a time (one cluster's solver CTA occupies an SM), the same
 * property that lets gdn_chunk_fwd callers share one workspace.
 */
gdn_status gdn_chunk_fwd_noalloc(const void *q, const void *k, const void *v, gdn_dtype in_dtype,
                                 const float *log_alpha, const float *beta, const float *S0,
                                 const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                                 int n_seq, int H, int d_k, int d_v, int chunk, float scale,
                                 void *y, gdn_dtype y_dtype, float *S_T, void *stream);

/*
 * gdn_selftest_bounded_wait -- runs the bounded mbarrier wait that every prefill-kernel
 * role uses, on the device, in one small CTA (failure handling; no counterpart in the
 * pages). Thread 0 waits on a barrier phase:
 *   mode 0: nothing completes it. After limit_cycles SM clocks the wait gives up and records
 *           GDN_ERR_TIMEOUT in the device error word, and the kernel exits normally.
 *   mode 1: another thread raises the kernel's abort flag after ~20K cycles. The wait returns
 *           at once and records nothing. limit_cycles >= 1e6 so that the abort comes first.
 *   mode 2: another thread completes the phase. The wait succeeds and records nothing.
 * A wait that returns the wrong answer for its mode records GDN_ERR_DEVICE_CHECK.
 * limit_cycles in [1, 2e9] (the kernels use 2e9, about 1 s). Asynchronous on `stream`; read
 * the outcome with gdn_device_error. GDN_ERR_INVALID_ARG for out-of-range arguments.
 */
gdn_status gdn_selftest_bounded_wait(int64_t limit_cycles, int mode, void *stream);

/*
 * gdn_chunk_fwd_gated -- gdn_chunk_fwd followed by the output epilogue in one call:
 * o = sigmoid(z) * RMSNorm(y) * (1 + w) per (token, head), as gdn_gate_norm defines it.
 * Two launches on the stream: the prefill writes y into o (in o_dtype), then the gate-norm
 * rewrites o in place. No buffer besides o and the workspace is used.
 *
 * Defines: the chunked prefill of gdn_chunk_fwd followed by the output-gate equation of
 * the joezjh.github.io notes ("GDN 参数化细节") with the zero-centred RMSNorm of the pwwt.cn
 * translation (section 2.1.1); the same arguments as gdn_chunk_fwd, plus
 *   z      [n_tok, H, d_v] bf16 (the projected gate logits)
 *   w      [d_v] fp32 (stored zero-centred weight; the scale is 1 + w);  eps >= 0 (1e-6)
 *   o      [n_tok, H, d_v] out, o_dtype (GDN_F32 or GDN_BF16), in place of y; it must not
 *          overlap z (GDN_ERR_INVALID_ARG, checked before any launch)
 * Only the tensor-core path: in_dtype GDN_BF16, d_k = d_v = 128, chunk = 64; anything else
 * returns GDN_ERR_UNSUPPORTED (call gdn_chunk_fwd then gdn_gate_norm). The workspace is
 * that of gdn_chunk_fwd. The result is bit-identical to gdn_chunk_fwd with y_dtype = o_dtype
 * followed by gdn_gate_norm of that y (so with GDN_BF16 o, y is rounded to bf16 first).
 * Errors: those of gdn_chunk_fwd, then those of gdn_gate_norm.
 */
gdn_status gdn_chunk_fwd_gated(const void *q, const void *k, const void *v, gdn_dtype in_dtype,
                               const float *log_alpha, const float *beta, const float *S0,
                               const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                               int n_seq, int H, int d_k, int d_v, int chunk, float scale,
                               const void *z, const float *w, float eps, void *o, gdn_dtype o_dtype,
                               float *S_T, void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdn_backward -- gradients of the chunked prefill's result with respect to its inputs.
 *
 * Defines: the reverse-mode adjoint of the token recurrence (joezjh.github.io notes,
 * "Gated DeltaNet 核心机制"; the pages report a backward kernel but print none) for
 * L = sum_t <dy_t, y_t> + <dS_T, S_T>:
 *   q, k, v, in_dtype, log_alpha, beta, S0, cu_seqlens_*, n_seq, H, d_k, d_v, scale: as for
 *          gdn_chunk_fwd (S0 may be NULL: zeros)
 *   dy     [n_tok, H, d_v] in in_dtype;  dS_T [n_seq, H, d_v, d_k] fp32 or NULL (zero)
 *   dq, dk [n_tok, H, d_k], dv [n_tok, H, d_v], dlog_alpha, dbeta [n_tok, H] fp32 out
 *          (dy, dq, dk, dv 16-byte aligned, like q, k, v)
 *   dS0    [n_seq, H, d_v, d_k] fp32 out, or NULL
 *   workspace: gdn_backward_workspace_bytes(...) bytes, 16-byte aligned: per (chain, chunk
 *          of 64 tokens) the chunk's start state and the adjoint of its end state
 *          (d_k x d_v each), its U~ and dU~ (64 x d_v each), the chunk's cache of state-free
 *          matrices (3 x 64 x 64 + 64 x d_k floats: T, A o Gamma, P, W) and, per slice of
 *          min(d_v, 64) value columns, one block of the chunk's sums over v
 *          (2 x 64 x 64 + 3 x 64 x d_k + 64 + 1 floats, rounded up to a multiple of 4);
 *          n_seq * H * ceil(max_len / 64) chunks are provided for
 *   d_k, d_v in {16, 32, 64, 128}
 * The chain rule through the chunked form, five launches, every matrix product on the
 * tensor cores with fp32-level accuracy (each operand split into two tf32 parts): the
 * state-free matrices of every chunk at once; a forward pass over the chunks of each
 * (chain, value slice) keeping each chunk's start state and U~; a reverse pass for the state
 * adjoints and dU~; then, for every chunk of every chain at once, dv and the per-slice sums
 * over v, and dq, dk, dbeta, dlog_alpha. Deterministic (no atomics).
 */
size_t gdn_backward_workspace_bytes(const int32_t *cu_seqlens_host, int n_seq, int H, int d_k,
                                    int d_v);
gdn_status gdn_backward(const void *q, const void *k, const void *v, gdn_dtype in_dtype,
                        const float *log_alpha, const float *beta, const float *S0,
                        const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host, int n_seq,
                        int H, int d_k, int d_v, float scale, const void *dy, const float *dS_T,
                        float *dq, float *dk, float *dv, float *dlog_alpha, float *dbeta, float *dS0,
                        void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdn_decode_step -- one token for each of n_seq * H independent chains, in place.
 *
 * Defines: the same four-line update (joezjh.github.io notes, "Gated DeltaNet 核心机制")
 * for a single token, with alpha given directly. It is computed in one pass over S:
 * with u = S^T k and r = S^T q taken on the old state, e = v - alpha u,
 * y = scale (alpha r + beta (k.q) e) (which equals S_new^T (scale q)), and
 * S <- alpha S + beta k e^T.
 *
 *   q, k   [n_seq, H, d_k] in in_dtype;  v [n_seq, H, d_v] in in_dtype
 *   alpha  [n_seq, H] fp32 in (0, 1];  beta [n_seq, H] fp32 in [0, 1]
 *   S      [n_seq, H, d_v, d_k] fp32, read and overwritten with the new state
 *   y      [n_seq, H, d_v] out, in y_dtype (GDN_F32 or GDN_BF16, independent of
 *          in_dtype; a bf16 y is the round-to-nearest-even of the fp32 result)
 *   d_k, d_v each in {16, 32, 64, 128}
 */
gdn_status gdn_decode_step(const void *q, const void *k, const void *v, gdn_dtype in_dtype,
                           const float *alpha, const float *beta, float *S, int n_seq, int H,
                           int d_k, int d_v, float scale, void *y, gdn_dtype y_dtype,
                           void *stream);

/*
 * gdn_decode_tokens -- n_tokens consecutive tokens for each of n_seq * H chains, in place,
 * in one pass over the state (the multi-token decode of speculative decoding).
 *
 * Defines: the update of gdn_decode_step applied token after token (joezjh.github.io
 * notes, "Gated DeltaNet 核心机制"); the result equals n_tokens calls of gdn_decode_step.
 * The state is read and written once per call, so the HBM cost per token falls by
 * n_tokens. Token i of sequence s is row (s * n_tokens + i) of the inputs:
 *
 *   q, k   [n_seq * n_tokens, H, d_k] in in_dtype;  v [n_seq * n_tokens, H, d_v] in in_dtype
 *   alpha  [n_seq * n_tokens, H] fp32 in (0, 1];  beta [n_seq * n_tokens, H] fp32 in [0, 1]
 *   S      [n_seq, H, d_v, d_k] fp32, read and overwritten with the state after the last token
 *   y      [n_seq * n_tokens, H, d_v] out, in y_dtype (GDN_F32 or GDN_BF16, independent
 *          of in_dtype; a bf16 y is the round-to-nearest-even of the fp32 result)
 *   1 <= n_tokens <= 8; d_k, d_v each in {16, 32, 64, 128}
 * The pages run decode with several tokens per step (pwwt.cn translation, Figure 6
 * settings: next_n = 4) but give no kernel for it.
 */
gdn_status gdn_decode_tokens(const void *q, const void *k, const void *v, gdn_dtype in_dtype,
                             const float *alpha, const float *beta, float *S, int n_seq,
                             int n_tokens, int H, int d_k, int d_v, float scale, void *y,
                             gdn_dtype y_dtype, void *stream);

/*
 * gdn_gate_norm -- the output epilogue o = sigmoid(z) * RMSNorm(y) * (1 + w).
 *
 * Defines: the output-gate equation of the joezjh.github.io notes ("GDN 参数化细节")
 * without its W_z / W_o projections (z is the already projected gate logit), with the
 * zero-centred RMSNorm of the pwwt.cn translation (section 2.1.1): the stored weight
 * w multiplies as (1 + w); the input is not mean-subtracted. One row = one (token,
 * head); the mean is over its d_v elements.
 *
 *   y      [n_rows, d_v] in y_dtype;  z [n_rows, d_v] in z_dtype;  w [d_v] fp32
 *   o      [n_rows, d_v] out in o_dtype (each dtype GDN_F32 or GDN_BF16); o may be y itself
 *          (in place, y_dtype = o_dtype); otherwise o overlaps neither y nor z
 *          (GDN_ERR_INVALID_ARG, checked on the host before any launch)
 *   n_rows >= 0; d_v in {16, 32, 64, 128, 256}; eps > 0 recommended (1e-6)
 */
gdn_status gdn_gate_norm(const void *y, gdn_dtype y_dtype, const void *z, gdn_dtype z_dtype,
                         const float *w, int64_t n_rows, int d_v, float eps, void *o,
                         gdn_dtype o_dtype, void *stream);

/*
 * gdn_featurize -- the feature and gate step in front of the recurrence.
 *
 * Defines: the q/k/v and gate equations of the joezjh.github.io notes ("GDN 参数化细节")
 * with the projections W x given as inputs, and the pwwt.cn translation (section 2.1.1,
 * Figure 2): a short causal convolution of each projected stream, SiLU, then an L2 norm
 * of q and k (not v) per (token, head) over d:
 *   f_t = SiLU(sum_{j<W} conv[ch][j] * x_{t-(W-1)+j}),  x = 0 before the sequence start
 *   q_t = f_t / sqrt(|f_t|^2 + eps) (likewise k_t);  v_t = f_t
 *   beta_t = sigmoid(beta_logit_t);  log_alpha_t = -exp(A_h) * softplus(alpha_logit_t + b_alpha_h)
 * The window never reaches into an earlier sequence of the packed batch.
 *
 *   xq, xk [n_tok, H, d_k], xv [n_tok, H, d_v] in dtype (projected streams)
 *   conv_q, conv_k [H * d_k, W], conv_v [H * d_v, W] fp32 (tap j multiplies the row
 *          W - 1 - j tokens back: the layout of a depthwise Conv1d padded by W - 1)
 *   beta_logit, alpha_logit [n_tok, H] fp32;  A, b_alpha [H] fp32
 *   cu_seqlens_dev [n_seq + 1] int32 on the device, read by the kernels;
 *   cu_seqlens_host the same values on the host, or NULL (then unchecked here; tokens
 *          that the device copy does not cover raise GDN_ERR_DEVICE_CHECK)
 *   q, k [n_tok, H, d_k], v [n_tok, H, d_v] out, in dtype (the chunk_fwd inputs)
 *   beta, log_alpha [n_tok, H] out, fp32 (the chunk_fwd gates)
 *   d_k, d_v in {16, 32, 64, 128}; 1 <= W <= 4; eps >= 0 (1e-6; with eps = 0 an all-zero
 *   feature row gives NaN)
 * Outputs must not alias inputs. Two launches on `stream`, no synchronisation.
 * The pages do not give the convolution width or eps; there is no counterpart of
 * cu_seqlens on the pages (it delimits the packed sequences).
 */
gdn_status gdn_featurize(const void *xq, const void *xk, const void *xv, gdn_dtype dtype,
                         const float *conv_q, const float *conv_k, const float *conv_v, int W,
                         const float *beta_logit, const float *alpha_logit, const float *A,
                         const float *b_alpha, const int32_t *cu_seqlens_dev,
                         const int32_t *cu_seqlens_host, int n_seq, int64_t n_tok, int H, int d_k,
                         int d_v, float eps, void *q, void *k, void *v, float *beta,
                         float *log_alpha, void *stream);

/*
 * gdn_qsa_indexer -- the compressed lightweight indexer of Qwen Sparse Attention (QSA):
 * per query token, scores of the compressed key blocks and the K_B best blocks.
 *
 * Defines: the indexer equations of the joezjh.github.io notes page "Qwen3.8-Flash-Next"
 * (section on Qwen Sparse Attention, "压缩轻量级 Indexer": key compression, Partial RoPE,
 * block-causal ReLU importance, Top-K blocks) with the sizes of the pwwt.cn translation
 * (section on the QSA implementation: four indexer query heads sharing one key head,
 * token budget K = 2048 at compression ratio r = 4). The projections W x are inputs. For
 * each sequence of the packed batch (positions restart at its first token), with
 * RMSNorm(x) = x / sqrt(mean(x^2) + eps) * (1 + w) (zero-centred weight) and PRoPE(x, p)
 * rotating dimensions (j, j + rot/2), j < rot/2, by the angle p * base^(-2j/rot):
 *     q_i^h = PRoPE(RMSNorm_wq(qx_i^h), i)
 *     k_b   = PRoPE(RMSNorm_wk(mean_{j<r} kx_{b r + j}), b r)    b < n_b = floor(len / r)
 *     I_ib  = sum_h ReLU(<q_i^h, k_b>)      for the visible blocks b < nvis_i =
 *                                            min(n_b, floor((i + 1) / r))
 *     B_i   = the K_B = ceil(K / r) visible blocks of largest I_ib, ordered by score
 *             (descending) then block index (ascending, which also breaks ties); -1 padded
 *
 *   qx   [n_tok, Hq, d] and kx [n_tok, d] in dtype (GDN_BF16: tensor-core scores on bf16
 *        copies of the normalised, rotated vectors, fp32 accumulation; GDN_F32: fp32
 *        CUDA-core scores); wq, wk [d] fp32
 *   cu_seqlens_dev / cu_seqlens_host [n_seq + 1] int32 as for gdn_chunk_fwd
 *   Hq in {1, 2, 4} for GDN_BF16 (1..8 for GDN_F32); d = 128; r >= 1; K >= 1;
 *   rot even, 0 <= rot <= d; base > 0; eps >= 0
 *   scores  [n_tok, nb_max] fp32 out, nb_max = max over sequences of floor(len / r):
 *           I_ib for b < nvis_i; the other entries of a row are not written
 *   blocks  [n_tok, K_B] int32 out (B_i)
 *   workspace >= gdn_qsa_workspace_bytes(...) bytes, 16-byte aligned: the normalised,
 *           rotated queries and compressed keys
 * Four launches on `stream` (block and tile offsets, vectors, scores, selection). The pages
 * give no precision for the indexer; the selection is taken on the scores this call returns.
 */
size_t gdn_qsa_workspace_bytes(const int32_t *cu_seqlens_host, int n_seq, int Hq, int d, int r,
                               gdn_dtype dtype);
gdn_status gdn_qsa_indexer(const void *qx, const void *kx, gdn_dtype dtype, const float *wq,
                           const float *wk, const int32_t *cu_seqlens_dev,
                           const int32_t *cu_seqlens_host, int n_seq, int Hq, int d, int r, int K,
                           int rot, float base, float eps, float *scores, int32_t *blocks,
                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdn_qsa_token_sets -- the token set S_i of each query token from its selected blocks:
 * the r tokens of every selected block plus the tail r floor((i + 1) / r) .. i, in
 * ascending order (positions within the token's sequence), -1 padded.
 *
 * Defines: the final token set of the QSA indexer (joezjh.github.io notes, section on
 * Qwen Sparse Attention).
 *   blocks  [n_tok, K_B] int32 (gdn_qsa_indexer's output; -1 entries are skipped)
 *   tokens  [n_tok, K_B * r + r - 1] int32 out;  count [n_tok] int32 out (|S_i|)
 */
gdn_status gdn_qsa_token_sets(const int32_t *blocks, const int32_t *cu_seqlens_dev,
                              const int32_t *cu_seqlens_host, int n_seq, int K_B, int r,
                              int32_t *tokens, int32_t *count, void *stream);

/* A static, human-readable name for a status code. */
const char *gdn_status_string(gdn_status status);

/*
 * Synchronises `stream`, then reads and clears the current device's error word.
 * Returns GDN_OK, GDN_ERR_TIMEOUT or GDN_ERR_DEVICE_CHECK for conditions kernels
 * recorded, or GDN_ERR_CUDA if the synchronisation itself failed.
 */
gdn_status gdn_device_error(void *stream);

/* Library version as major * 10000 + minor * 100 + patch. */
int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
