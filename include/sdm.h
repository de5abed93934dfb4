/*
 * sdm.h -- C ABI of the B200 (sm_100a) Sparse Delta Memory recurrent core.
 *
 * The Sparse Delta Memory (SDM) layer keeps, per head, an explicit memory
 * M in R^{N x d_v} with N = sqrtN^2 slots. Per token it selects W write slots
 * and R read slots by product-key top-k, applies a gated delta write to the
 * write slots and reads a weighted sum of the read slots after the write.
 *
 * Sources (web pages about arXiv 2607.07386, "Sparse Delta Memory: Scaling the
 * State of Linear RNNs through Sparsity"):
 *   [explainer] papers.ananclaw.com explainer, section 3.1 "SDM 层的三步流程"
 *               (step 1 sparse key selection, step 2 gated delta write,
 *               step 3 sparse read), section 3.2 (isoFLOP), section 3.3 (eq. 6);
 *   [summary]   gist.science "Technical Summary: Sparse Delta Memory (SDM)",
 *               Methodology / Core Mechanism items 1-4.
 *
 * Conventions for every entry point:
 *   - Pointers named as tensors are caller-owned DEVICE pointers to contiguous
 *     row-major arrays, 16-byte aligned (alpha and beta: aligned to their
 *     element size). The library allocates no memory; scratch space is passed
 *     in by the caller ("workspace").
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream). Calls only enqueue work and return; results are ready when the
 *     stream reaches them.
 *   - Argument errors are detected on the host before anything is enqueued and
 *     return SDM_ERR_INVALID_ARGUMENT / SDM_ERR_UNSUPPORTED; sdm_last_error()
 *     then names the argument. A failed kernel launch returns SDM_ERR_CUDA.
 *     Problems found on the device (an index outside [0, N), a bounded wait
 *     that expired) set a per-device error word that sdm_stream_check()
 *     reports as SDM_ERR_DEVICE_FAULT; such entries are skipped, never
 *     dereferenced.
 *   - Shapes: B batch rows, T tokens, H heads; a "token-head" is one (b,t,h).
 *     Index order in [B,T,H,X] arrays is b slowest, X fastest.
 *   - dtype SDM_F32 is IEEE binary32, SDM_BF16 is bfloat16 (round-to-nearest-
 *     even on every store).
 *   - Not thread-safe with respect to one stream; distinct streams may call
 *     concurrently. Library-wide state: the per-device error word, the
 *     thread-local message behind sdm_last_error(), and per-device caches
 *     made on first use (device attributes, the scratch address of
 *     sdm_layer_forward_noalloc, the two streams of an overlapped
 *     sdm_layer_forward call). The caches do not survive cudaDeviceReset():
 *     reload the library after a reset. The error word is
 *     shared by all streams of a device: sdm_stream_check() on any stream
 *     reports (and clears) the bits set by every stream's calls since the last
 *     check, so a multi-stream caller should check after a common sync point.
 *   - A bounded wait that expires (kernels wait at most ~2 s on their own
 *     copies) stops its thread block; copies it had in flight may still land
 *     in shared memory that a later block on the same SM then uses, so after a
 *     wait-timeout report every output of every call since the last check is
 *     undefined and must be discarded, not only the tile that timed out.
 */
#ifndef SDM_B200_SDM_H_
#define SDM_B200_SDM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SDM_ABI_VERSION 2

#if defined(__GNUC__)
#define SDM_API __attribute__((visibility("default")))
#else
#define SDM_API
#endif

typedef enum sdm_status {
  SDM_OK = 0,
  SDM_ERR_INVALID_ARGUMENT = 1, /* a null pointer, a size out of range, misalignment */
  SDM_ERR_UNSUPPORTED = 2,      /* valid but outside what the kernels implement */
  SDM_ERR_CUDA = 3,             /* a CUDA runtime call or launch failed */
  SDM_ERR_DEVICE_FAULT = 4      /* the device error word was set (see sdm_stream_check) */
} sdm_status_t;

/* SDM_FP8_B16 is a state dtype only: OCP FP8 E4M3 codes with one
 * power-of-two scale per 16 consecutive values of a state row. A state of
 * R rows of d_v values is R * d_v code bytes followed by R * d_v / 16 int8
 * exponents (value = E4M3(code) * 2^exponent); sdm_quantize_fp8blk builds it
 * from fp32 (for M0 [H,N,d_v]: H*N rows; M [B,H,N,d_v]: B*H*N rows, so M's
 * codes of every batch row come first, then their exponents). It runs in the
 * single-launch decode step (sdm_layer_step with T = 1, W = R <= 64,
 * automatic variant) and in the pipelined recurrence (sdm_scan,
 * sdm_layer_forward, sdm_layer_step with T > 1; automatic or pipelined
 * variant; d_v a multiple of 256, so that a row's exponents fill 16-byte
 * rows), which applies the write to each decoded 16-value block in fp32 and
 * re-quantises it exactly as the decode step does. Other variants and the
 * backward return SDM_ERR_UNSUPPORTED for it. */
typedef enum sdm_dtype { SDM_F32 = 0, SDM_BF16 = 1, SDM_FP8_B16 = 2 } sdm_dtype_t;

/* Which recurrence kernel runs (sdm_shape_t.variant). */
typedef enum sdm_variant {
  SDM_VARIANT_AUTO = 0,      /* pick by size: resident when the state tile fits, pipelined
                                when 128-byte column tiles leave SMs idle (and for the fp8
                                state), else streaming */
  SDM_VARIANT_RESIDENT = 1,  /* the (b,h) state column tile lives in shared memory */
  SDM_VARIANT_STREAMING = 2, /* the state stays in global memory; rows are gathered
                                ahead of use and scattered back */
  SDM_VARIANT_PIPELINED = 3  /* as streaming, for few (b,h) sequences: each column tile's
                                slots are split over two CTAs (more SMs moving rows),
                                and each CTA's warps split writes, reads and gathers */
} sdm_variant_t;

/* One layer call.
 *   B, T, H   >= 0 (T == 0 is a no-op apart from state initialisation)
 *   sqrt_n    in [1, 1024]; N = sqrt_n * sqrt_n slots per head
 *   W, R      write / read slots per token-head, in [1, min(N, 256)]
 *   d_v       columns per slot, a multiple of 16, <= 8192
 *   in_dtype    dtype of k', q', v, alpha, beta, g
 *   state_dtype dtype of M0, M (the recurrence computes in fp32 and rounds on store)
 *   rms_eps   epsilon of the optional RMS-norm epilogue
 *   variant   an sdm_variant_t value
 *   tile      0: the library picks the kernel's tile; k in [1, 64]: use the k-th
 *             entry of the chosen kernel's tile table among those that fit this
 *             shape (sdm_scan_describe names it; SDM_ERR_UNSUPPORTED if there is
 *             no k-th). For measurements: the state comes out the same, y the
 *             same up to the order of its fp32 sums. In the backward with
 *             shared-memory tiles, 1 selects one warp per tile. */
typedef struct sdm_shape {
  int32_t B, T, H;
  int32_t sqrt_n;
  int32_t W, R;
  int32_t d_v;
  int32_t in_dtype;
  int32_t state_dtype;
  float rms_eps;
  int32_t variant;
  int32_t tile;
} sdm_shape_t;

/* ABI version of the loaded library (SDM_ABI_VERSION). */
SDM_API int32_t sdm_abi_version(void);

/* Static text for a status code. */
SDM_API const char* sdm_status_string(sdm_status_t status);

/* Text describing the last error returned on the calling host thread ("" if none). */
SDM_API const char* sdm_last_error(void);

/* Quantises n_blocks blocks of 16 fp32 values into the SDM_FP8_B16 format:
 * codes = round-to-nearest-even(x / 2^e) onto the E4M3 grid, with e per block
 * the smallest integer for which that rounding of max|x| / 2^e is at most 448
 * (i.e. max|x| <= 464 * 2^e; clamped to [-127, 127]; 0 for an all-zero
 * block), so no value saturates and re-quantising a decoded block returns it
 * unchanged. x [n_blocks * 16] fp32; codes [n_blocks * 16] uint8;
 * exps [n_blocks] int8 (all device, caller owned; x and codes 16-byte aligned). */
SDM_API sdm_status_t sdm_quantize_fp8blk(const float* x, int64_t n_blocks, uint8_t* codes, int8_t* exps,
                                 void* stream);

/* Slot utilisation of a selection: counts[b,h,i] += the number of (t,k) with
 * idx[b,t,h,k] == i ([explainer] "亮点与局限" and "工程落地关键点" item 2: the
 * learned addressing can collapse onto few slots, so the per-slot update
 * frequencies are worth tracking; the pages give no kernel for it).
 *   idx    [B,T,H,K] int32 (e.g. the write slots of sdm_pkm_topk)
 *   counts [B,H,N] int32, accumulated (zero it first; calls over consecutive
 *          token ranges add up). Indices outside [0, N) are skipped and set the
 *          device error word. */
SDM_API sdm_status_t sdm_slot_counts(const int32_t* idx, int32_t B, int32_t T, int32_t H, int32_t K,
                             int32_t N, int32_t* counts, void* stream);

/* Product-key top-k selection ([explainer] 3.1 step 1; [summary] Core Mechanism 2).
 * For every token-head, x = scores[b,t,h,:] is split into s1 = x[0:sqrt_n] and
 * s2 = x[sqrt_n:2*sqrt_n]. Slot i = a*sqrt_n + b has score s1[a] + s2[b]. The K
 * slots first in the order (exact real sum descending, slot ascending) are
 * found via topk(s1 (+) s2) = topk(topk(s1) (+) topk(s2)) without forming the N
 * sums; -0 and +0 are equal. The weights are the softmax of the K selected
 * scores, each score rounded to fp32 (the pages leave these weights undefined;
 * this is the reading the library implements).
 *   scores  [B,T,H,2*sqrt_n] in_dtype (NaN gives an unspecified but in-range selection)
 *   idx_out [B,T,H,K] int32, slots in selection order
 *   w_out   [B,T,H,K] fp32, softmax weights aligned with idx_out
 *   K in [1, min(N, 256)]. */
SDM_API sdm_status_t sdm_pkm_topk(const void* scores, int32_t in_dtype, int32_t B, int32_t T, int32_t H,
                          int32_t sqrt_n, int32_t K, int32_t* idx_out, float* w_out, void* stream);

/* Bytes of workspace sdm_scan needs for this shape (0 for invalid shapes). */
SDM_API size_t sdm_scan_workspace_bytes(const sdm_shape_t* shape);

/* The recurrence kernel sdm_scan / sdm_layer_forward would run for this shape
 * on the current device: SDM_VARIANT_RESIDENT, SDM_VARIANT_STREAMING or
 * SDM_VARIANT_PIPELINED, or -1 if the shape is invalid or unsupported
 * (sdm_last_error() says why). */
SDM_API int32_t sdm_scan_variant(const sdm_shape_t* shape);

/* The launch configuration of that kernel as text, e.g.
 * "resident CW=8 NWARP=1 L=4 EB=4 smem=...",
 * "streaming C=64 P=3 L=8 NW=16 smem=..." or
 * "pipelined C=64 P=6 L=16 NWW=4 NWR=3 NP=8 S=1 parts=2 smem=...", NUL-terminated into out (caller
 * owned, out_len bytes, truncated to fit). Returns SDM_OK, or an error for an
 * invalid or unsupported shape (out left empty). For profiles and logs. */
SDM_API sdm_status_t sdm_scan_describe(const sdm_shape_t* shape, char* out, size_t out_len);

/* Bytes of workspace sdm_scan_backward needs for this shape (0 if the shape is
 * invalid or the backward does not support it; sdm_last_error() says why). */
SDM_API size_t sdm_scan_backward_workspace_bytes(const sdm_shape_t* shape);

/* Backward of sdm_scan (no epilogue): the derivatives a training step needs
 * ([explainer] 3.4 "高效训练" says that a memory-efficient backward exists; the
 * derivatives follow from 3.1 steps 2-3 by the chain rule, for a fixed
 * selection). For the loss L with dy = dL/dy and dM = dL/dM_T it computes,
 * with a_i = alpha_t (1 - beta_t k_i), c_i = beta_t k_i, G = dL/dM_t:
 *   dq_j     = <dy_t, M_t[j]>                        -> dw_r
 *   dk_i     = beta_t (<G[i], v_t> - alpha_t <G[i], M_{t-1}[i]>)  -> dw_w
 *   dv_t     = sum_i c_i G[i]
 *   dalpha_t = sum_i (1 - beta_t k_i) <G[i], M_{t-1}[i]>
 *   dbeta_t  = sum_i k_i (<G[i], v_t> - alpha_t <G[i], M_{t-1}[i]>)
 *   dM       <- dL/dM_0 (in place)
 * The state trajectory is recomputed from M_in (checkpoints every C tokens
 * plus a log of overwritten rows, all in the workspace), bit-identical to the
 * forward's. Requires an fp32 state (state_dtype SDM_F32), else
 * SDM_ERR_UNSUPPORTED. While 4-column tiles of the state and its adjoint fit
 * in shared memory (N up to about 6900) they stay there (C = 128); larger
 * states use 32-column tiles in global memory (a working copy of the state in
 * the workspace, dM updated in place) with C near sqrt(T N / W).
 *   idx_w, w_w, idx_r, w_r, v, alpha, beta: the forward's inputs (as sdm_scan)
 *   M_in  fp32, the state the forward started from: [B,H,N,d_v], or [H,N,d_v]
 *         shared by every batch row when m_in_shared != 0
 *   dy    [B,T,H,d_v] fp32 (the derivative of the pre-epilogue y)
 *   dM    [B,H,N,d_v] fp32, in: dL/dM_T (zeros if the final state is unused),
 *         out: dL/dM_0 per batch row (sum over b for a shared M_0)
 *   dv    [B,T,H,d_v] fp32; dalpha, dbeta [B,T,H] fp32; dw_w [B,T,H,W] fp32;
 *   dw_r  [B,T,H,R] fp32 (all written, caller owned)
 *   workspace: device scratch of sdm_scan_backward_workspace_bytes(shape).
 * Results are deterministic. Slot indices outside [0, N) are skipped and set
 * the device error word. */
SDM_API sdm_status_t sdm_scan_backward(const sdm_shape_t* shape, const int32_t* idx_w, const float* w_w,
                               const int32_t* idx_r, const float* w_r, const void* v, const void* alpha,
                               const void* beta, const float* M_in, int32_t m_in_shared, const float* dy,
                               float* dM, float* dv, float* dalpha, float* dbeta, float* dw_w, float* dw_r,
                               void* workspace, size_t workspace_bytes, void* stream);

/* The RMS-norm x gate epilogue alone, in place ([explainer] 3.1 step 3):
 * y <- g * y / sqrt(mean(y^2) + eps) over each of n_rows rows of d_v.
 *   y [n_rows, d_v] fp32 (in/out); g [n_rows, d_v] in in_dtype (SDM_F32 or
 *   SDM_BF16). sdm_layer_forward applies the same epilogue when given g;
 *   training keeps the row before it (y_pre) by running the layer without g
 *   and this afterwards. */
SDM_API sdm_status_t sdm_rmsnorm_gate(float* y, const void* g, int32_t in_dtype, int64_t n_rows, int32_t d_v,
                              float eps, void* stream);

/* Sum of squares of each of n_rows rows of d_v fp32 values, in a fixed order:
 * ss[r] = sum_c y[r, c]^2. When the d_v columns of a layer call are split
 * across devices (each device holding a column slice of every row), the sum of
 * the devices' ss is the full rows' sum that the RMS-norm epilogue needs
 * ([explainer] 3.1 step 3); one all-reduce of ss per call combines them.
 *   y [n_rows, d_v] fp32;  ss [n_rows] fp32 out (caller owned). */
SDM_API sdm_status_t sdm_row_sumsq(const float* y, int64_t n_rows, int32_t d_v, float* ss, void* stream);

/* The RMS-norm x gate epilogue on a column slice: for n_rows rows of a layer
 * output with d_total columns of which this slice holds d_v,
 * y <- g * y / sqrt(ss / d_total + eps), with ss the full rows' sums of
 * squares (e.g. sdm_row_sumsq summed over the devices).
 *   y [n_rows, d_v] fp32 (in/out); g [n_rows, d_v] in in_dtype; ss [n_rows] fp32. */
SDM_API sdm_status_t sdm_rmsnorm_gate_rows(float* y, const void* g, int32_t in_dtype, const float* ss, int64_t n_rows,
                                           int32_t d_v, int32_t d_total, float eps, void* stream);

/* Backward of the epilogue for dout = dL/dout, with x = y_pre (the row
 * before it), r = sqrt(mean(x^2) + eps):
 *   dy_pre_j = g_j dout_j / r - x_j sum_i(g_i dout_i x_i) / (d_v r^3)
 *   dg_i     = dout_i x_i / r
 * y_pre, dout, dy_pre, dg: [n_rows, d_v] fp32; g in in_dtype. */
SDM_API sdm_status_t sdm_rmsnorm_gate_backward(const float* y_pre, const void* g, int32_t in_dtype,
                                       const float* dout, int64_t n_rows, int32_t d_v, float eps,
                                       float* dy_pre, float* dg, void* stream);

/* Bytes of workspace sdm_layer_backward needs (0 if unsupported; see
 * sdm_scan_backward). */
SDM_API size_t sdm_layer_backward_workspace_bytes(const sdm_shape_t* shape);

/* Backward of the whole layer as sdm_layer_forward computes it with a shared
 * initial state M0 [H,N,d_v] fp32: re-selects the slots of kp and qp
 * (sdm_pkm_topk), then the epilogue's backward when g is given
 * (sdm_rmsnorm_gate_backward on y_pre), the recurrence's
 * (sdm_scan_backward), and both selection-weight backwards
 * (sdm_pkm_topk_backward).
 *   dy     [B,T,H,d_v] fp32: dL/d(layer output)
 *   y_pre  [B,T,H,d_v] fp32: the layer output before the epilogue (only with g)
 *   dM     [B,H,N,d_v] fp32: in dL/dM_T (zeros if unused), out dL/dM0 per
 *          batch row (sum over b for M0's gradient)
 *   dkp, dqp [B,T,H,2*sqrt_n]; dv [B,T,H,d_v]; dalpha, dbeta [B,T,H];
 *   dg [B,T,H,d_v] (only with g): fp32 outputs, caller owned.
 * Needs an fp32 state (shape.state_dtype SDM_F32). */
SDM_API sdm_status_t sdm_layer_backward(const sdm_shape_t* shape, const void* kp, const void* qp, const void* v,
                                const void* alpha, const void* beta, const void* g, const float* M0,
                                const float* y_pre, const float* dy, float* dM, float* dkp, float* dqp,
                                float* dv, float* dalpha, float* dbeta, float* dg, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Checkpoints of the recurrence for a later backward of the same call, so
 * that the backward need not recompute them ([explainer] 3.4: the memory-
 * efficient backward recomputes the forward from stored states): the state
 * before tokens C, 2C, ..., (n-1)C, n = ceil(T / C), as [n-1][B,H,N,d_v]
 * fp32, where C (*chunk_tokens) is the checkpoint chunk sdm_layer_backward
 * uses for this shape. Sets *bytes (0 when T <= C). SDM_ERR_UNSUPPORTED when
 * the forward does not store them for this shape: only the resident
 * recurrence with an fp32 state does (the backward then recomputes them). */
SDM_API sdm_status_t sdm_layer_checkpoint_size(const sdm_shape_t* shape, int32_t* chunk_tokens, size_t* bytes);

/* sdm_layer_forward that also writes those checkpoints into ckpt (device,
 * 16-byte aligned, at least the bytes sdm_layer_checkpoint_size reports;
 * caller owned). Same results as sdm_layer_forward, bit for bit. */
SDM_API sdm_status_t sdm_layer_forward_ckpt(const sdm_shape_t* shape, const void* kp, const void* qp, const void* v,
                                    const void* alpha, const void* beta, const void* g, const void* M0,
                                    void* M_out, float* y, float* ckpt, size_t ckpt_bytes, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* sdm_layer_backward given the checkpoints sdm_layer_forward_ckpt stored for
 * the same inputs (or NULL: recompute them): the recurrence backward then
 * skips its first pass over the tokens. Same results, bit for bit (the
 * forward's states are the states the backward recomputes). */
SDM_API sdm_status_t sdm_layer_backward_ckpt(const sdm_shape_t* shape, const void* kp, const void* qp, const void* v,
                                     const void* alpha, const void* beta, const void* g, const float* M0,
                                     const float* y_pre, const float* dy, float* dM, float* dkp, float* dqp,
                                     float* dv, float* dalpha, float* dbeta, float* dg, const float* ckpt,
                                     size_t ckpt_bytes, void* workspace, size_t workspace_bytes, void* stream);

/* Backward of the selection weights of sdm_pkm_topk for a fixed selection
 * ([explainer] 3.1 step 1: w = softmax of the K selected sums
 * sigma_k = s1[a_k] + s2[b_k], slot a_k * sqrt_n + b_k):
 *   dsigma_k = w_k (dw_k - sum_j w_j dw_j);  dscores[a_k] += dsigma_k;
 *   dscores[sqrt_n + b_k] += dsigma_k;  other entries 0.
 *   idx, w, dw [B,T,H,K] (int32, fp32, fp32): the selection, its weights and
 *              dL/dw;  dscores [B,T,H,2*sqrt_n] fp32 out (caller owned).
 * Deterministic (fixed summation order). Indices outside [0, N) are skipped
 * and set the device error word. */
SDM_API sdm_status_t sdm_pkm_topk_backward(const int32_t* idx, const float* w, const float* dw, int32_t B,
                                   int32_t T, int32_t H, int32_t sqrt_n, int32_t K, float* dscores,
                                   void* stream);

/* The sparse gated delta recurrence over a given selection, in token order
 * ([explainer] 3.1 steps 2-3; [summary] Core Mechanism 3-4). For each token t
 * and head: for every write slot i (distinct within a token),
 *     M[i] <- M~ + beta_t * k_i * (v_t - M~),  M~ = alpha_t * M[i]
 * (computed as (alpha_t*(1 - beta_t*k_i)) * M[i] + (beta_t*k_i) * v_t in fp32),
 * other slots untouched; then y_t = sum_r q_r * M[r] over the read slots, on
 * the updated state. With g != NULL, y_t <- g_t * y_t / sqrt(mean(y_t^2) + rms_eps).
 *   idx_w, w_w [B,T,H,W] int32 / fp32;  idx_r, w_r [B,T,H,R] int32 / fp32
 *   v     [B,T,H,d_v] in_dtype;  alpha, beta [B,T,H] in_dtype
 *   g     [B,T,H,d_v] in_dtype or NULL
 *   M     [B,H,N,d_v] state_dtype, read as M_0 and overwritten with M_T, so calls
 *         over consecutive token ranges chain exactly
 *   y     [B,T,H,d_v] fp32 output
 *   workspace: device scratch of at least sdm_scan_workspace_bytes(shape), 16-byte
 *         aligned, not read before it is written.
 * Write indices repeated within one token-head give unspecified values. */
SDM_API sdm_status_t sdm_scan(const sdm_shape_t* shape, const int32_t* idx_w, const float* w_w,
                      const int32_t* idx_r, const float* w_r, const void* v, const void* alpha,
                      const void* beta, const void* g, void* M, float* y, void* workspace,
                      size_t workspace_bytes, void* stream);

/* M[b] <- M0 for every batch row b (the learned initial state of the
 * [explainer] 3.1 "learned initial state" paragraph, shared by all rows).
 *   M0 [H,N,d_v] state_dtype;  M [B,H,N,d_v] state_dtype. */
SDM_API sdm_status_t sdm_state_init(const sdm_shape_t* shape, const void* M0, void* M, void* stream);

/* Bytes of workspace sdm_layer_forward needs for this shape (0 for invalid shapes). */
SDM_API size_t sdm_layer_forward_workspace_bytes(const sdm_shape_t* shape);

/* One SDM layer core: selection on k' (top-W) and q' (top-R), M_out <- M0 for
 * every batch row, the recurrence, and the optional epilogue.
 *   kp, qp [B,T,H,2*sqrt_n] in_dtype;  v, alpha, beta, g as in sdm_scan
 *   M0     [H,N,d_v] state_dtype (not modified);  M_out [B,H,N,d_v] state_dtype (M_T)
 *   y      [B,T,H,d_v] fp32
 *   workspace: at least sdm_layer_forward_workspace_bytes(shape).
 * Overlapped call: with one batch row (B = 1), the pipelined recurrence and
 * T >= 131072, the call runs as chunks of 65536 tokens (sdm_layer_forward_chunks):
 * the selection of the next chunk runs on the SMs the recurrence leaves free
 * while the recurrence of the current chunk runs, on two streams the library
 * creates per device (one at the greatest, one at the least priority). They
 * start after the work enqueued on `stream` before the call, and `stream`
 * waits for all of their work, so to the caller the call is ordered on
 * `stream` as any other. The outputs are those of the one-pass call bit for bit
 * (the recurrence over consecutive chunks continues from the state in M_out;
 * selection and records are per token). */
SDM_API sdm_status_t sdm_layer_forward(const sdm_shape_t* shape, const void* kp, const void* qp,
                               const void* v, const void* alpha, const void* beta, const void* g,
                               const void* M0, void* M_out, float* y, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Kernel launches one sdm_layer_forward call makes for this shape on the
 * current device (with_gate != 0: with the epilogue): the two selections,
 * the record build and the recurrence, plus the state copy for the streaming
 * and pipelined recurrences, plus the pass that adds the second slot part's
 * read sums into y (pipelined, two parts), plus the epilogue. -1 for an
 * invalid or unsupported shape. For profiles and logs. */
SDM_API int32_t sdm_layer_forward_launches(const sdm_shape_t* shape, int32_t with_gate);

/* Token chunks one sdm_layer_forward call runs this shape as on the current
 * device: 1 for a one-pass call, more for an overlapped call (see
 * sdm_layer_forward); each chunk makes two selections, a record build and a
 * recurrence launch. -1 for an invalid or unsupported shape. */
SDM_API int32_t sdm_layer_forward_chunks(const sdm_shape_t* shape);

/* Kernel launches one sdm_layer_step call makes for this shape, without the
 * epilogue's (one more when g is given on the general path): 1 when the call
 * takes the single-launch decode kernel (T = 1, W = R <= 64, automatic
 * variant), else 4 (two selections, records, recurrence).
 * -1 for an invalid shape. For profiles and logs. */
SDM_API int32_t sdm_layer_step_launches(const sdm_shape_t* shape);

/* Bytes of workspace sdm_layer_step needs for this shape (0 for invalid shapes). */
SDM_API size_t sdm_layer_step_workspace_bytes(const sdm_shape_t* shape);

/* One call of the layer core that carries the state across calls (the
 * decode / streaming use: T = 1 or a few tokens per call): selection on k'
 * (top-W) and q' (top-R), the recurrence starting from the state in M, and the
 * optional epilogue ([explainer] 3.1 steps 1-3). M [B,H,N,d_v] state_dtype is
 * read as the state before the first token and overwritten with the state
 * after the last, so consecutive calls over consecutive token ranges continue
 * one sequence (start from M[b] = M0 with sdm_state_init). Other arguments as
 * in sdm_layer_forward; workspace: at least sdm_layer_step_workspace_bytes(shape).
 * With the automatic variant, calls with T*(W+R) < N stream only the selected
 * rows (a resident tile would move the whole state), and calls with T = 1 and
 * W = R <= 64 run as one fused launch (both selections, the write, the read
 * and the epilogue). The fp8 state (state_dtype SDM_FP8_B16: M is the code
 * bytes followed by the block exponents, as sdm_quantize_fp8blk writes them)
 * runs in that fused form and, for T > 1, in the pipelined recurrence. */
SDM_API sdm_status_t sdm_layer_step(const sdm_shape_t* shape, const void* kp, const void* qp,
                            const void* v, const void* alpha, const void* beta, const void* g,
                            void* M, float* y, void* workspace, size_t workspace_bytes, void* stream);

/* sdm_layer_forward that also records caller-created CUDA events (cudaEvent_t
 * passed as void*) on `stream` between its stages, for timing each kernel in
 * place: events[0] before the selection on k', [1] after the selection on q',
 * [2] after the record build, [3] after the state initialisation, [4] after
 * the recurrence kernel, [5] after the epilogue (a stage that does not run
 * leaves its event adjacent to the previous one). n_events must be 0 (no
 * events; events may be NULL) or 6. In an overlapped call the events go on
 * the library's streams: [1] and [2] after the first chunk's selection and
 * records, [3] before the first chunk's recurrence, [4] after the last
 * chunk's recurrence and the part sum, [5] after the epilogue; there
 * n_events may also be 6 + 2 * sdm_layer_forward_chunks(shape), and
 * events[6 + 2k] and events[7 + 2k] are recorded right before and after the
 * recurrence launch of chunk k (the recurrence kernel's own time). */
SDM_API sdm_status_t sdm_layer_forward_traced(const sdm_shape_t* shape, const void* kp, const void* qp,
                                      const void* v, const void* alpha, const void* beta,
                                      const void* g, const void* M0, void* M_out, float* y,
                                      void* workspace, size_t workspace_bytes, void* stream,
                                      void* const* events, int32_t n_events);

/* sdm_layer_forward for callers that cannot hand the library any device
 * memory for scratch -- for example a plugin inside a host engine that owns
 * the whole device pool and offers no workspace, or a latency-bound loop that
 * must not call an allocator after start-up (cudaMalloc can synchronise the
 * device and stall). The caller still passes every input and output; the
 * scratch comes from one array of SDM_NOALLOC_SCRATCH_BYTES (16 MiB) that the
 * library keeps in device memory on every GPU that loads it, until the
 * process exits. Nothing is allocated or freed here.
 *   - Shapes whose sdm_layer_forward_workspace_bytes() exceeds
 *     SDM_NOALLOC_SCRATCH_BYTES are rejected with SDM_ERR_INVALID_ARGUMENT.
 *   - The first call on a device looks up the array's device address (a
 *     one-time set-up per device); make that first call before any stream
 *     capture.
 *   - All calls on a device share the one array and it keeps what the last
 *     call left there (no part of it needs to start at zero). Calls whose work
 *     overlaps on the GPU -- on different streams, or from different host
 *     threads -- race on it; order them on one stream.
 * The paper has no counterpart to this entry point; it is an interface for
 * such hosts. Arguments and results are as in sdm_layer_forward. */
#define SDM_NOALLOC_SCRATCH_BYTES (16u << 20)
SDM_API sdm_status_t sdm_layer_forward_noalloc(const sdm_shape_t* shape, const void* kp, const void* qp,
                                       const void* v, const void* alpha, const void* beta,
                                       const void* g, const void* M0, void* M_out, float* y,
                                       void* stream);

/* Waits for `stream`, then reads and clears the current device's error word
 * (shared by all streams of the device; see the conventions above).
 * Returns SDM_ERR_DEVICE_FAULT if it was set (sdm_last_error() gives the bits
 * in hex and names them), SDM_ERR_CUDA if the synchronisation failed, else
 * SDM_OK. */
SDM_API sdm_status_t sdm_stream_check(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SDM_B200_SDM_H_ */
