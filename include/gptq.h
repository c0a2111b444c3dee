/*
 * gptq.h — C ABI of the B200 (sm_100a) GPTQ per-layer quantization solve.
 *
 * The method (quantize one linear layer W [m x n] from calibration activations X [N x n]):
 *   S1  H += 2 X^T X over calibration batches
 *       ("模型量化实战：从 INT8 PTQ 到 GPTQ 的精度保持与推理加速全解析", §3.2, accumulate_hessian)
 *   S2  dead columns (diag H == 0): H_ii = 1 and the weight column is zeroed;
 *       damping H += damp * mean(diag H) * I  (same page, §3.2 prepare)
 *   S3  act-order (desc_act): columns sorted by descending diag H
 *       ("GPTQ量化损失深度解析：原理、影响与优化策略", 减少量化损失的实战策略)
 *   S4  U = upper Cholesky factor of H^-1 (H^-1 = U^T U)   (§3.2 prepare)
 *   S5  column sweep in blocks of 128: per-group min-max scale/zero, b-bit code,
 *       e = (w - q) / U[i,i], W[:, j>i] -= e * U[i, j]
 *       ("大模型量化：GPTQ/AWQ/GGUF 原理对比，4-bit 量化对推理精度的影响", GPTQ section)
 *   S6  the later columns of W are updated once per 128-column block by one product
 *   S7  codes packed per row, scales, zeros, perm and g_idx
 *
 * Conventions (all calls):
 *   - Every tensor pointer is CALLER-OWNED DEVICE memory on the context's device unless the
 *     argument says otherwise; the context owns only its workspace.
 *   - All matrices are row-major with the leading dimension stated.
 *   - Calls are enqueued on the context's CUDA stream and return after launching, except
 *     gptq_prepare and gptq_synchronize, which wait (with a bounded host wait) for the stream.
 *   - Arguments are validated on the host before anything is launched; a call that returns
 *     an error other than GPTQ_ERR_CUDA / GPTQ_ERR_TIMEOUT has enqueued nothing.
 *   - Device-side failures (a non-positive pivot, a kernel wait that ran out) are recorded
 *     in a device status word and returned by the next gptq_prepare / gptq_synchronize.
 *   - There is no CPU fallback: without a CUDA device every compute call fails with
 *     GPTQ_ERR_CUDA.
 */
#ifndef GPTQ_B200_H
#define GPTQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct gptq_ctx gptq_ctx; /* opaque: device H, factor, permutation and workspace */

typedef enum {
  GPTQ_OK = 0,
  GPTQ_ERR_ARG = 1,         /* invalid argument (null pointer, size, alignment, range) */
  GPTQ_ERR_STATE = 2,       /* call not allowed in the context's current state */
  GPTQ_ERR_NOT_PD = 3,      /* damped Hessian not positive definite (non-positive pivot) */
  GPTQ_ERR_OOM = 4,         /* workspace does not fit (checked before allocating) */
  GPTQ_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed (no device, launch error...) */
  GPTQ_ERR_TIMEOUT = 6,     /* a bounded device or host wait ran out */
  GPTQ_ERR_UNSUPPORTED = 7  /* valid request that this library does not implement */
} gptq_status;

/* Quantizer settings ("GPTQ算法原理深度解析" §3.3 quantize_config: bits, group_size; sym from
 * "GPTQ量化损失深度解析" 调整量化参数).
 *   bits       : 2, 3, 4 or 8.
 *   group_size : columns per scale/zero group, in sweep order; -1 = one group per row
 *                (per-channel).  Must divide n and either divide 128 or be a multiple of
 *                128; at least 32.
 *   sym        : 0 = asymmetric min-max (range widened to include 0; zero-point integer in
 *                [0, 2^b-1]); 1 = symmetric (scale = max|w| / (2^(b-1)-1), signed codes stored
 *                offset by 2^(b-1), zero = 2^(b-1)).
 * Dequantization is always (code - zero) * scale. */
typedef struct {
  int bits;
  int group_size;
  int sym;
} gptq_qparams;

/* Device bytes a context for n_in input features and at most m_max output rows allocates
 * (H, damped H, V, U, the inverse temporary, the fp32 working copy of W and small buffers).
 * Returns 0 for sizes that gptq_create rejects.  Pure host function. */
size_t gptq_workspace_bytes(int64_t n_in, int64_t m_max);

/* Create a context for layers with n_in input features (n_in % 128 == 0, 128 <= n_in <= 32768)
 * and up to m_max output rows (1 <= m_max <= 2^24).  `device` is the CUDA ordinal;
 * `cuda_stream` is a cudaStream_t (NULL = legacy default stream) that every later call of
 * this context is enqueued on.  Allocates the whole workspace up front: returns GPTQ_ERR_OOM
 * without allocating when gptq_workspace_bytes() exceeds the device's free memory or the
 * limit in the environment variable GPTQ_MAX_WORKSPACE_BYTES.  H starts at zero.
 * On success *out owns the workspace until gptq_destroy. */
gptq_status gptq_create(gptq_ctx** out, int64_t n_in, int64_t m_max, int device, void* cuda_stream);

/* S1: H += 2 X^T X for one calibration batch and n_tok += batch size (asynchronous).
 *   X_bf16 : device, bf16, [n_tok x n_in] row-major with leading dimension ld_x elements
 *            (ld_x >= n_in, ld_x % 8 == 0, 16-byte aligned base).
 *   n_tok  : tokens in this batch, 0 <= n_tok < 2^31 (0 is a no-op).
 * Runs the tcgen05 BF16 x BF16 -> FP32 accumulator.  GPTQ_ERR_STATE after gptq_prepare
 * until gptq_reset. */
gptq_status gptq_hessian_accumulate(gptq_ctx* ctx, const void* X_bf16, int64_t n_tok, int64_t ld_x);

/* Copy the accumulated H (full symmetric, fp32, [n x n], leading dimension n) to the device
 * buffer H_out and the token count to the HOST int64 *n_tok_out (either may be NULL).
 * Waits for the context's stream. */
gptq_status gptq_get_hessian(gptq_ctx* ctx, float* H_out, int64_t* n_tok_out);

/* Replace H by a caller-provided symmetric fp32 [n x n] device matrix (leading dimension n)
 * and set the token count (resumes a saved calibration).  Only the upper triangle is read.
 * GPTQ_ERR_STATE after gptq_prepare until gptq_reset. */
gptq_status gptq_set_hessian(gptq_ctx* ctx, const float* H_in, int64_t n_tok);

/* S2-S4 (synchronizes once): dead-column fix, optional act-order permutation, damping by
 * damp * mean(diag H) (0 <= damp <= 1e6), then U = upper-Cholesky(H_perm^-1) by a blocked
 * reverse Cholesky H_perm = V V^T and U = V^-1.  Past 1024 columns only the blocks of U the
 * sweep reads are formed here (V whole, U inside every aligned 1024-column diagonal block and
 * inside the recursion's right parts); gptq_get_factor forms the rest when asked.
 *   desc_act : 0 = identity order; 1 = stable descending diag H (after the dead fix).
 *   perm_out : device int32 [n] or NULL; perm_out[k] = original column swept at position k.
 * Returns GPTQ_ERR_NOT_PD when a pivot is not positive (the context stays unprepared).
 * H itself is left unchanged, so prepare may be repeated with another damp. */
gptq_status gptq_prepare(gptq_ctx* ctx, double damp, int desc_act, int32_t* perm_out);

/* Copy the factor U (fp32 [n x n], sweep order, zeros below the diagonal) to the device
 * buffer U_out.  The first call after a gptq_prepare of a layer wider than 1024 columns first
 * launches the products that complete U (up to about 40 % of the factorization's work);
 * later results of gptq_quantize_layer do not change.  GPTQ_ERR_STATE before gptq_prepare.
 * Asynchronous. */
gptq_status gptq_get_factor(gptq_ctx* ctx, float* U_out);

/* Copy the dead-column mask of the last gptq_prepare to the device buffer dead_out
 * (uint8 [n], ORIGINAL column order): 1 where diag(H) was 0, so that the column was treated
 * as unexcited (H_ii = 1) and its weights are zeroed by gptq_quantize_layer; 0 elsewhere.
 * This is the `dead` input gptq_quantize_layer_noalloc needs to reproduce the context's
 * result.  GPTQ_ERR_STATE before gptq_prepare.  Asynchronous. */
gptq_status gptq_get_dead_columns(gptq_ctx* ctx, uint8_t* dead_out);

/* S5-S7 (asynchronous): quantize W with the prepared factor.
 *   W_fp16     : device fp16 [m x n] row-major (ld n), ORIGINAL column order, 1 <= m <= m_max.
 *   codes_out  : device uint32 [m x n*bits/32]; row r holds its codes in SWEEP order as an
 *                LSB-first bit stream (code k in stream bits k*bits .. k*bits+bits-1, stream bit
 *                p = bit p%32 of word p/32).
 *   scales_out : device fp32 [m x G], G = n / group_size (1 for per-channel), groups in sweep
 *                order.
 *   zeros_out  : device fp32 [m x G], integer-valued.
 *   g_idx_out  : device int32 [n] or NULL; g_idx[perm[k]] = k / group_size.
 *   W_hat_out  : device fp32 [m x n] or NULL; dequantized weights in ORIGINAL column order.
 * The columns past each slab of the sweep receive the slab's contribution as (W0 - Q) Vs
 * with Vs = V blockdiag(U_SS), which the first call after gptq_prepare forms (one product);
 * group widths that do not fit a power-of-two slab of at most 1024 columns use -E U on the
 * completed factor instead (the same arithmetic in exact numbers).
 * GPTQ_ERR_STATE before gptq_prepare. */
gptq_status gptq_quantize_layer(gptq_ctx* ctx, const void* W_fp16, int64_t m, gptq_qparams qp,
                                uint32_t* codes_out, float* scales_out, float* zeros_out,
                                int32_t* g_idx_out, float* W_hat_out);

/* Wait (bounded by GPTQ_SYNC_TIMEOUT_MS, default 600000) for the context's stream and return
 * the first recorded device-side failure, if any. */
gptq_status gptq_synchronize(gptq_ctx* ctx);

/* Zero H and the token count and return to the accumulate state (asynchronous). */
gptq_status gptq_reset(gptq_ctx* ctx);

/* Free the workspace (waits for the stream).  NULL is accepted. */
gptq_status gptq_destroy(gptq_ctx* ctx);

/* Number of kernels this context has launched since gptq_create (instrumentation; -1 for
 * NULL).  Pure host function. */
int64_t gptq_launch_count(const gptq_ctx* ctx);

/* Allocation-free variant of gptq_quantize_layer for callers that cannot allocate device
 * memory themselves (a host that owns a fixed device-memory budget, or code that must not
 * call cudaMalloc/cudaFree, which synchronize the device).  The page has no counterpart:
 * it is a deployment convenience, not a step of the method.
 * It runs the S5-S7 kernels with their scratch (the fp32 working copy of W and the
 * per-block error tile) in a fixed array compiled into this library, so it calls no
 * cudaMalloc, cudaFree or other allocating routine:
 *   - the array holds 2^20 fp32 working weights plus 4096 x 128 fp32 errors (6 MiB); every
 *     GPU that loads the library keeps it until the process exits;
 *   - limits: m <= 4096, m * n <= 2^20, 128 <= n <= 32768 with n % 128 == 0; larger requests
 *     return GPTQ_ERR_ARG before anything is launched;
 *   - every call shares the one array (it keeps the last call's contents; nothing in it has
 *     to start at zero), so calls that overlap on the GPU — on different streams, or from
 *     different host threads — race and corrupt each other; serialize them;
 *   - the first call on a device resolves the array's device address (and raises kernel
 *     shared-memory limits) with that device current; make that first call before any
 *     stream capture.
 * Inputs (device): W_fp16 [m x n] fp16, original column order; U [n x n] fp32 upper factor
 * in sweep order (as from gptq_get_factor); perm [n] int32 (as from gptq_prepare); dead
 * [n] uint8 (1 = dead column, weights zeroed) or NULL for none.  Outputs as in
 * gptq_quantize_layer.  `device` is the CUDA ordinal, `cuda_stream` a cudaStream_t the
 * kernels are enqueued on (asynchronous). */
gptq_status gptq_quantize_layer_noalloc(const void* W_fp16, int64_t m, int64_t n, const float* U,
                                        const int32_t* perm, const uint8_t* dead, gptq_qparams qp,
                                        uint32_t* codes_out, float* scales_out, float* zeros_out,
                                        int32_t* g_idx_out, float* W_hat_out, int device, void* cuda_stream);

/* ---------------------------------------------------------------------------------------
 * Many layers in one call, pipelined ("大模型量化：GPTQ/AWQ/GGUF 原理对比…", AWQ vs GPTQ section:
 * quantizing a whole 7B model layer by layer takes hours on one A100; here the per-layer solves
 * of a block overlap on one GPU).
 *
 * Each job is one layer: its calibration activations, its weights, its quantizer settings and
 * its outputs (the arguments of gptq_hessian_accumulate, gptq_prepare and gptq_quantize_layer):
 *   X_bf16, n_tok, ld_x : device bf16 [n_tok x n] calibration activations (leading dimension ld_x)
 *   W_fp16, m, n        : device fp16 [m x n] weights, original column order
 *   qp, damp, desc_act  : quantizer settings and prepare settings
 *   codes_out, scales_out, zeros_out, g_idx_out (may be NULL), perm_out (device int32 [n], may
 *   be NULL), W_hat_out (may be NULL): as in gptq_prepare / gptq_quantize_layer.
 * Jobs whose X_bf16, n_tok, ld_x and n are equal share one Hessian (e.g. the q, k and v
 * projections of a transformer block read the same input); within such a group, jobs with the
 * same damp and desc_act share one factorization.  Groups run in order of first appearance on
 * two internal contexts and streams: the Hessian and the factorization of group i run while the
 * quantization of group i-1 runs.  The call allocates its contexts (two per distinct width n;
 * GPTQ_ERR_OOM before any launch if they do not fit), waits for `cuda_stream` before starting,
 * returns once every job is done (bounded waits) and frees the contexts.
 * Returns the first error (GPTQ_ERR_NOT_PD names no job; the outputs of later jobs are then
 * undefined). */
typedef struct {
  const void* X_bf16;
  int64_t n_tok, ld_x;
  const void* W_fp16;
  int64_t m, n;
  gptq_qparams qp;
  double damp;
  int desc_act;
  uint32_t* codes_out;
  float* scales_out;
  float* zeros_out;
  int32_t* g_idx_out;
  int32_t* perm_out;
  float* W_hat_out;
} gptq_layer_job;

gptq_status gptq_quantize_layers(const gptq_layer_job* jobs, int count, int device, void* cuda_stream);

/* The same pipeline with its contexts kept between calls (gptq_quantize_layers creates and frees
 * them on every call).  gptq_pipeline_create allocates two contexts for each of the `count`
 * distinct widths widths[i] (up to m_max[i] rows each; GPTQ_ERR_OOM before allocating if they
 * do not fit) and two streams; each gptq_pipeline_run waits for `cuda_stream` (the stream given
 * at create) before starting, quantizes its jobs as gptq_quantize_layers does (GPTQ_ERR_ARG if
 * a job's width has no context or its m exceeds that width's m_max) and returns when they are
 * done.  Group i of a run (jobs sharing an input) runs on the two contexts alternately: its
 * Hessian and factorization overlap the quantization of group i-1.  gptq_pipeline_destroy
 * waits for the streams and frees everything (NULL is accepted).  A pipeline is used by one
 * host thread at a time. */
typedef struct gptq_pipeline gptq_pipeline;
gptq_status gptq_pipeline_create(gptq_pipeline** out, const int64_t* widths, const int64_t* m_max, int count,
                                 int device, void* cuda_stream);
gptq_status gptq_pipeline_run(gptq_pipeline* pipeline, const gptq_layer_job* jobs, int count);
gptq_status gptq_pipeline_destroy(gptq_pipeline* pipeline);

/* ---------------------------------------------------------------------------------------
 * AWQ on the same calibration activations and weights
 * ("大模型量化：GPTQ/AWQ/GGUF 原理对比，4-bit 量化对推理精度的影响", AWQ section):
 *   importance[c] = mean_t |X[t][c]|      (summed in fp64)
 *   scale[c]      = s_protect if importance[c] > median(importance) else 1
 *                   (median of an even count: the lower of the two middle values)
 *   W'            = fp32(W) * scale[c]     (each input channel)
 *   codes, scales, zeros: round-to-nearest of W' with the min-max groups of gptq_qparams in
 *                   ORIGINAL column order (no act-order, no error compensation); codes packed
 *                   LSB-first per row as in gptq_quantize_layer
 *   W_hat         = (code - zero) * group scale / scale[c]   (optional)
 * At inference the activations are divided by scale[c].  s_protect = 1 is plain round-to-
 * nearest.  X_bf16: device bf16 [n_tok x n] (ld_x >= n, ld_x % 8 == 0, 16-byte aligned;
 * n_tok may be 0: every scale is 1); W_fp16: device fp16 [m x n]; channel_scale_out: device
 * fp32 [n]; workspace: device, 256-byte aligned, gptq_awq_workspace_bytes(n) bytes (fp64 channel
 * sums and the median).  Asynchronous on cuda_stream; arguments checked before any launch. */
size_t gptq_awq_workspace_bytes(int64_t n);
gptq_status gptq_awq_quantize(const void* X_bf16, int64_t n_tok, int64_t ld_x, const void* W_fp16, int64_t m, int64_t n,
                              float s_protect, gptq_qparams qp, uint32_t* codes_out, float* scales_out,
                              float* zeros_out, float* channel_scale_out, float* W_hat_out, void* workspace,
                              size_t workspace_bytes, int device, void* cuda_stream);

/* ---------------------------------------------------------------------------------------
 * Round-to-nearest with a clipped range
 * ("模型量化实战：从 INT8 PTQ 到 GPTQ 的精度保持与推理加速全解析" §3.1, LinearQuantizer and its
 *  clip_ratio: outliers are clipped so that the rest of the weights get a finer step.)
 *   W'      = fp32(W) * channel_scale[c]   (channel_scale may be NULL: 1; pass the scales of
 *             gptq_awq_quantize to clip an AWQ-scaled layer)
 *   range   per row and group of gptq_qparams (ORIGINAL column order):
 *             clip_ratio = 1: min and max of W' (max |W'| for sym), as gptq_awq_quantize;
 *             clip_ratio < 1, sym:  the 100 c-th percentile of |W'|;
 *                             asym: the (1 - c) 50-th and 100 - (1 - c) 50-th percentiles of W'
 *             A percentile is the linear interpolation between the order statistics of ranks
 *             floor(h) and floor(h) + 1 at h = (g - 1) q, in fp32 as numpy computes it for fp32
 *             data: q = fp32(p) / 100, t = h - floor(h), a + (b - a) t for t < 1/2, else
 *             b - (b - a)(1 - t).
 *   scale, zero from the range as in gptq_quantize_layer (asym range widened to include 0,
 *             scales floored at 1e-8); codes clip(round_half_even(W' / s + z)), so the weights
 *             outside the range saturate; packed LSB-first per row in original column order.
 *   W_hat   = (code - zero) * group scale / channel_scale[c]   (optional, may be NULL)
 * W_fp16: device fp16 [m x n] (n % 128 == 0, 128 <= n <= 32768); codes_out: device uint32
 * [m x n*bits/32]; scales_out, zeros_out: device fp32 [m x n/g]; clip_ratio in (0, 1], else
 * GPTQ_ERR_ARG.  Every pointer is caller-owned device memory.  Asynchronous on cuda_stream;
 * arguments checked before any launch. */
gptq_status gptq_rtn_quantize(const void* W_fp16, int64_t m, int64_t n, gptq_qparams qp, float clip_ratio,
                              const float* channel_scale, uint32_t* codes_out, float* scales_out, float* zeros_out,
                              float* W_hat_out, int device, void* cuda_stream);

/* ---------------------------------------------------------------------------------------
 * The packed result's consumer: Y = X W16^T
 * ("模型量化实战：从 INT8 PTQ 到 GPTQ 的精度保持与推理加速全解析" §4.3: INT4 weights are turned
 *  back into FP16 before the matrix product; the low-bit storage saves memory bandwidth.)
 *
 *   W16[r][k] = fp16( fp32(code[r][k] - zero[r][k / g]) * scale[r][k / g] )   (sweep order k)
 *   Y[t][r]   = sum_k X[t][perm[k]] * W16[r][k]      (fp16 products, fp32 accumulation)
 *
 * gptq_dequant_matmul_workspace_bytes: device bytes of caller-provided workspace the call
 *   needs for T tokens, m output rows and n input features (act_order: 1 when a perm is
 *   passed); 0 for sizes the call rejects.  Pure host function.
 * gptq_dequant_matmul (asynchronous, on cuda_stream):
 *   X_fp16    : device fp16 [T x n] row-major, ORIGINAL column order, 16-byte aligned;
 *               1 <= T <= 2^24
 *   codes     : device uint32 [m x n*bits/32], scales/zeros: device fp32 [m x G], exactly as
 *               gptq_quantize_layer writes them (16-byte aligned codes)
 *   perm      : device int32 [n] (sweep position k holds original column perm[k]) or NULL for
 *               the identity order
 *   qp        : bits and group_size as quantized (sym is encoded in the zeros and not read)
 *   Y         : device fp32 [T x m] row-major output
 *   workspace : device, 256-byte aligned, at least gptq_dequant_matmul_workspace_bytes; holds a
 *               status word, the activations gathered into sweep order and split-K partial
 *               sums; owned by the caller, may be reused by later calls on the same stream
 *   n % 128 == 0, 128 <= n <= 2^20, 1 <= m <= 2^24.  Arguments are checked before any launch
 *   (GPTQ_ERR_ARG); the result is deterministic (split-K partials are summed in a fixed order).
 * gptq_dequant_matmul_check: waits (bounded) for cuda_stream and returns GPTQ_ERR_TIMEOUT if
 *   a bounded wait of the last gptq_dequant_matmul on this workspace ran out, else GPTQ_OK. */
size_t gptq_dequant_matmul_workspace_bytes(int64_t T, int64_t m, int64_t n, int act_order);
gptq_status gptq_dequant_matmul(const void* X_fp16, int64_t T, const uint32_t* codes, const float* scales,
                                const float* zeros, const int32_t* perm, int64_t m, int64_t n, gptq_qparams qp,
                                float* Y, void* workspace, size_t workspace_bytes, int device, void* cuda_stream);
gptq_status gptq_dequant_matmul_check(void* workspace, int device, void* cuda_stream);

/* ---------------------------------------------------------------------------------------
 * Sequential (cross-layer) quantization ("GPTQ算法原理深度解析" §2.1: the quantization error of a
 * layer reaches the next layer through its input): layer l+1 is calibrated on the outputs of
 * the already-quantized layer l, y = X_l W16_l^T (gptq_dequant_matmul), through the model's
 * activation.  This call forms those inputs:
 *   x = act(y)   act 0 = identity, 1 = ReLU (y if y > 0, else 0)
 *   Y        : device, `count` values, fp32 (in_bf16 = 0) or bf16 (in_bf16 = 1)
 *   out_bf16 : device bf16 [count] or NULL (the next Hessian's input), round to nearest even
 *   out_fp16 : device fp16 [count] or NULL (the next product's input), round to nearest even
 * At least one output.  Asynchronous on cuda_stream. */
gptq_status gptq_activation_convert(const void* Y, int in_bf16, int64_t count, int act, void* out_bf16, void* out_fp16,
                                    int device, void* cuda_stream);

/* Per-kernel instrumentation (off by default).  While profiling is on, every kernel the
 * context launches is bracketed by CUDA timing events on the context's stream and the
 * factorization runs as individual launches instead of its recorded graph (so launches no
 * longer overlap their predecessor: totals are slightly above those of normal runs).
 * gptq_get_profile waits for the stream (bounded), folds the records into one entry per
 * kernel role and clears them.
 *   name     : kernel and role, e.g. "gemm_tf32x3:factor"
 *   launches : launches recorded
 *   ms       : sum of the launches' event durations
 *   flops    : algorithmic floating-point operations of those launches (the product's nonzero
 *              multiply-adds x 2, counted once however many partial products the kernel forms;
 *              0 for kernels that are not contractions)
 *   bytes    : algorithmic bytes read and written by those launches (0 where not stated)
 * gptq_get_profile writes at most `capacity` entries to the host array `out` and the number
 * of roles recorded to *count (which may exceed capacity). */
typedef struct {
  char name[40];
  int64_t launches;
  double ms;
  double flops;
  double bytes;
} gptq_kernel_stat;

gptq_status gptq_set_profiling(gptq_ctx* ctx, int on);
gptq_status gptq_get_profile(gptq_ctx* ctx, gptq_kernel_stat* out, int capacity, int* count);

/* Static description of a status code. */
const char* gptq_status_string(gptq_status s);

/* Tokens per tensor-memory accumulation chunk of S1 (a multiple of 64).  Each chunk is
 * summed on the tensor cores, then added to fp32 running sums with round-to-nearest adds,
 * which bounds the accumulation error of long calibration sets.  Default 512. */
gptq_status gptq_set_hessian_chunk(gptq_ctx* ctx, int64_t tokens);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_H */
