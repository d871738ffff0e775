/*
 * sq.h -- C ABI of the SmoothQuant W8A8 linear layer for NVIDIA B200 (sm_100a).
 *
 * What the library computes (source pages cited by title and section):
 *
 *   [SQ-depth] "SmoothQuant, in depth: where the scales fold, how calibration
 *              feeds them, and a W8A8 pipeline you can ship"
 *   [LLMint8]  "LLM.int8() and SmoothQuant"
 *
 *   1. calibration: per input channel j, the running max over calibration
 *      tokens of |x_j| at a smoothed Linear's input ([SQ-depth] "The
 *      calibration data flow");
 *   2. smoothing factors s_j = max|X_j|^alpha / max|W_j|^(1-alpha), shared by
 *      all Linears that read one norm, and the fold of 1/s into that norm's
 *      gamma (and beta) ([LLMint8] "Fix 2" and "going deeper"; [SQ-depth]
 *      "Where the scales go in a decoder block");
 *   3. smoothed weights diag(s) W quantised to INT8 with one scale per output
 *      channel ([LLMint8] "going deeper"; [SQ-depth] "Granularity");
 *   4. at run time: the norm (carrying 1/s) and a per-token dynamic absmax
 *      INT8 quantisation of its output ([SQ-depth] "Granularity");
 *   5. an INT8 x INT8 GEMM with exact INT32 accumulation and an epilogue
 *      out = acc * scale_token[i] * scale_channel[j] emitted as bf16
 *      ([SQ-depth] "Granularity"; "The problem SmoothQuant solves").
 *
 * Around that path:
 *   - inputs with no norm in front, still quantised per token ([SQ-depth]
 *     "Where the scales go in a decoder block"): a ReLU GEMM output whose row
 *     maxima the GEMM epilogue reduces (sq_w8a8_gemm_dequant_rowmax, then
 *     sq_quant_per_token_given_absmax), and SiLU(gate) * up of a merged
 *     gate/up projection quantised in one pass (sq_silu_mul_quant_per_token);
 *   - one scale per tensor (the O2 / O3 levels of [SQ-depth] "Granularity"):
 *     sq_norm_smooth_absmax, sq_norm_smooth_quant_per_tensor,
 *     sq_smooth_quantize_weights_per_tensor;
 *   - FP8 (e4m3) codes with the same smoothing ([LLMint8] "example . what you
 *     get"): sq_norm_smooth_quant_per_token_fp8, sq_smooth_quantize_weights_fp8,
 *     sq_silu_mul_quant_per_token_fp8, sq_fp8_gemm_dequant;
 *   - the row split of a Linear over several GPUs (exact collectives between
 *     the calls): sq_row_absmax, sq_dequant_i32;
 *   - LLM.int8()'s decomposition as a comparator on the same inputs
 *     ([LLMint8] "Fix 1"): sq_llmint8_outliers, sq_llmint8_combine;
 *   - planning and allocation-free variants: sq_w8a8_gemm_plan,
 *     sq_w8a8_gemm_workspace_size, sq_w8a8_gemm_dequant_noalloc; the two
 *     halves of step 2 (sq_weight_column_max, sq_smooth_scales_from_maxima).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Layout: activations are row-major [M, K] (M tokens, K input channels) with
 *   a row stride ld (elements); weights are nn.Linear-shaped row-major [N, K]
 *   (N output channels); outputs are row-major [M, N] with stride ldo.
 * - Memory: every tensor pointer is DEVICE memory owned by the caller.  Except
 *   where a call says otherwise the library allocates nothing and frees
 *   nothing.  Pointer arguments marked "host" are host memory read during the
 *   call only.
 * - Execution: every call enqueues work on `stream` (a cudaStream_t; NULL is
 *   the legacy default stream) and returns without synchronising.  Calls keep
 *   no state between them and may be made from several threads.
 * - Arithmetic: rounding is IEEE round-to-nearest-even everywhere; INT8 codes
 *   are symmetric, clamped to [-127, 127]; a row whose absmax is 0 gets scale 0
 *   and codes 0.  Results are bit-identical from run to run.
 * - Alignment: input tensor and parameter-vector base pointers must be
 *   16-byte aligned and K and every input row stride ld must keep rows 16-byte
 *   aligned (K % 16 == 0 for the INT8 tensors, ld % 8 == 0 for bf16 rows,
 *   ld % 4 == 0 for fp32 rows); otherwise the call returns SQ_ERR_ALIGNMENT
 *   and launches nothing.  GEMM outputs need only element alignment: rows
 *   that are 16-byte aligned are written with 128-bit stores, others element
 *   by element.
 * - Errors: arguments are checked on the host before anything is launched; a
 *   failing call returns a non-zero sq_status and leaves its outputs
 *   untouched.  Faults the GPU can only discover later (a pipeline wait that
 *   ran out) are recorded in a device error word that sq_get_device_error()
 *   reads.  No call aborts the process.
 */
#ifndef SQ_H_
#define SQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SQ_OK = 0,
  SQ_ERR_INVALID_ARG = 1,      /* NULL pointer, negative size, bad enum, ld < K */
  SQ_ERR_UNSUPPORTED = 2,      /* dtype / shape this build does not handle */
  SQ_ERR_ALIGNMENT = 3,        /* pointer or row stride not 16-byte aligned */
  SQ_ERR_OVERFLOW_RISK = 4,    /* K so large that 127*127*K could overflow INT32 */
  SQ_ERR_CUDA = 5,             /* a CUDA runtime call or launch failed */
  SQ_ERR_PIPELINE_TIMEOUT = 6, /* a device-side wait gave up (read later) */
  SQ_ERR_WORKSPACE = 7         /* workspace missing or smaller than required */
} sq_status;

typedef enum { SQ_F32 = 0, SQ_BF16 = 1 } sq_dtype;

typedef enum { SQ_NORM_NONE = 0, SQ_NORM_RMS = 1, SQ_NORM_LAYER = 2 } sq_norm;

typedef enum {
  SQ_EPI_BF16 = 0,      /* out bf16 = bf16(fp32(fp32(float(acc) * xs[m]) * ws[n])) */
  SQ_EPI_BF16_RELU = 1, /* the same with max(., 0) before the bf16 rounding */
  SQ_EPI_I32_RAW = 2,   /* out int32 = acc (no scaling; for exactness checks) */
  SQ_EPI_F32_RAW = 3    /* FP8 GEMMs only: out fp32 = the fp32 accumulator */
} sq_epilogue;

/* Largest K for which |sum_k q_a q_b| <= 127*127*K fits in INT32. */
#define SQ_MAX_K 133144

/*
 * sq_calibrate_absmax -- running per-channel absmax of the norm output.
 * [SQ-depth] "The calibration data flow": record, for every smoothed Linear,
 * the running maximum over all calibration tokens of |x_j| at its input,
 * combining batches with an element-wise maximum.  The Linear's input is the
 * output of its (unsmoothed) norm: y = norm(x; gamma, beta, eps).
 *   x        device [M, K] with row stride ldx, fp32 or bf16 (dtype)
 *   norm     SQ_NORM_RMS, SQ_NORM_LAYER, or SQ_NORM_NONE (y = x, or
 *            y = x * gamma when gamma is given)
 *   gamma    device [K] fp32, or NULL for gamma = 1
 *   beta     device [K] fp32, or NULL for beta = 0 (LayerNorm only)
 *   eps      norm epsilon, added to the mean square / variance in fp64
 *   act_max  device [K] fp32, IN/OUT: act_max[j] = max(act_max[j],
 *            max_m |y[m, j]|).  The caller zero-fills it before the first
 *            batch.  M == 0 is a no-op.
 * Errors: SQ_ERR_INVALID_ARG, SQ_ERR_ALIGNMENT, SQ_ERR_CUDA.
 */
sq_status sq_calibrate_absmax(const void* x, sq_dtype dtype, int64_t M, int64_t K,
                              int64_t ldx, sq_norm norm, const float* gamma,
                              const float* beta, float eps, float* act_max, void* stream);

/*
 * sq_compute_smooth_scales -- smoothing factors and the folded norm.
 * [LLMint8] "going deeper": s_j = max_t|X_tj|^alpha / max|W_j|^(1-alpha);
 * [SQ-depth] "Where the scales go in a decoder block": all Linears reading one
 * norm share one s from the element-wise maximum of their weights, and gamma
 * (and beta) are divided by s; [SQ-depth] "The calibration data flow": both
 * maxima are clamped below at clamp_eps before the powers, s itself after.
 *   act_max   device [K] fp32 (from sq_calibrate_absmax)
 *   W         HOST array of num_w DEVICE pointers, weight l is [N[l], K]
 *             row-major (stride K), all of one dtype
 *   N         HOST array of num_w output sizes
 *   alpha     migration strength in [0, 1]
 *   clamp_eps lower clamp of both maxima and of s (1e-5 on the page)
 *   gamma     device [K] fp32 norm weight, or NULL for gamma = 1 (a Linear
 *             with no norm in front: gamma_folded = 1/s is then applied as a
 *             per-channel multiplier by SQ_NORM_NONE)
 *   beta      device [K] fp32 or NULL
 *   s         device [K] fp32 OUT: fl32 of the fp64 value
 *             max(max(a,eps)^alpha / max(w,eps)^(1-alpha), eps); it is also
 *             used as scratch during the call
 *   gamma_folded  device [K] fp32 OUT: fl32(gamma / s)
 *   beta_folded   device [K] fp32 OUT or NULL: fl32(beta / s)
 * Errors: SQ_ERR_INVALID_ARG (alpha outside [0,1], num_w < 1, ...),
 *         SQ_ERR_ALIGNMENT, SQ_ERR_CUDA.
 */
sq_status sq_compute_smooth_scales(const float* act_max, const void* const* W,
                                   const int64_t* N, int num_w, sq_dtype dtype, int64_t K,
                                   double alpha, float clamp_eps, const float* gamma,
                                   const float* beta, float* s, float* gamma_folded,
                                   float* beta_folded, void* stream);

/*
 * The two halves of sq_compute_smooth_scales, for callers that overlap the
 * weight column maxima (which need no calibration data) with calibration:
 *
 * sq_weight_column_max -- w_max[j] = max over the num_w weights l and their
 * rows n of |W_l[n, j]| (the weights exactly widened to fp32).
 *   W, N, num_w, dtype, K  as for sq_compute_smooth_scales
 *   w_max     device [K] fp32 OUT (zeroed by the call on the stream first)
 * Errors: SQ_ERR_INVALID_ARG, SQ_ERR_ALIGNMENT, SQ_ERR_UNSUPPORTED, SQ_ERR_CUDA.
 */
sq_status sq_weight_column_max(const void* const* W, const int64_t* N, int num_w, sq_dtype dtype,
                               int64_t K, float* w_max, void* stream);

/*
 * sq_smooth_scales_from_maxima -- s, gamma_folded and beta_folded of
 * sq_compute_smooth_scales from both maxima: act_max (sq_calibrate_absmax)
 * and w_max (sq_weight_column_max).  s may be w_max itself (updated in place).
 * Other arguments and errors as for sq_compute_smooth_scales.
 */
sq_status sq_smooth_scales_from_maxima(const float* act_max, const float* w_max, int64_t K,
                                       double alpha, float clamp_eps, const float* gamma,
                                       const float* beta, float* s, float* gamma_folded,
                                       float* beta_folded, void* stream);

/*
 * sq_smooth_quantize_weights -- W-hat = W diag(s), INT8 per output channel.
 * [LLMint8] "going deeper": W-hat = diag(s) W (column j of an nn.Linear
 * weight times s_j), then quantised per channel; [SQ-depth] "Granularity":
 * per-output-channel weight scales.
 *   W      device [N, K] row stride ldw, fp32 or bf16
 *   s      device [K] fp32, or NULL for an unsmoothed Linear (s = 1)
 *   Wq     device [N, K] int8 OUT (dense, stride K)
 *   w_scale device [N] fp32 OUT: fl32(max_k |W-hat[n,k]| / 127)
 * Codes: Wq = clamp(rne(fl32(W-hat / w_scale)), -127, 127).
 * Errors: SQ_ERR_INVALID_ARG, SQ_ERR_ALIGNMENT, SQ_ERR_CUDA.
 */
sq_status sq_smooth_quantize_weights(const void* W, sq_dtype dtype, int64_t N, int64_t K,
                                     int64_t ldw, const float* s, int8_t* Wq, float* w_scale,
                                     void* stream);

/*
 * sq_norm_smooth_quant_per_token -- fused norm (with the folded 1/s) and
 * per-token dynamic absmax INT8 quantisation.
 * [SQ-depth] "Where the scales go in a decoder block": the norm with gamma/s
 * (and beta/s) emits X/s with no extra kernel; [SQ-depth] "Granularity":
 * per-token dynamic activation scales; [LLMint8] "Try it": step = max / 127.
 *   x        device [M, K] row stride ldx, fp32 or bf16
 *   norm     SQ_NORM_RMS / SQ_NORM_LAYER, or SQ_NORM_NONE for a Linear with
 *            no norm in front (y = x, or x * gamma_folded when given)
 *   gamma_folded device [K] fp32 or NULL (= 1)
 *   beta_folded  device [K] fp32 or NULL (= 0; LayerNorm only)
 *   Xq       device [M, K] int8 OUT (dense, stride K)
 *   x_scale  device [M] fp32 OUT: fl32(max_k |y[m,k]| / 127)
 * Norm arithmetic: row sums of x and x^2 in fp64, then
 *   RMS:  r = fl32(1 / sqrt(S2/K + eps));  y = fl32(fl32(x r) gamma)
 *   LN:   mu = S1/K, var = max(0, S2/K - mu^2), r = fl32(1/sqrt(var + eps)),
 *         y = fl32(fl32(fl32(fl32(x - fl32(mu)) r) gamma) + beta)
 * (every fp64 step is one IEEE operation).
 * Errors: SQ_ERR_INVALID_ARG, SQ_ERR_ALIGNMENT, SQ_ERR_UNSUPPORTED (K too
 *         large for one CTA per row), SQ_ERR_CUDA.
 */
sq_status sq_norm_smooth_quant_per_token(const void* x, sq_dtype dtype, int64_t M, int64_t K,
                                         int64_t ldx, sq_norm norm, const float* gamma_folded,
                                         const float* beta_folded, float eps, int8_t* Xq,
                                         float* x_scale, void* stream);

/*
 * Per-tensor variants (the paper's O2 and O3 levels).
 * [SQ-depth] "Granularity: O1, O2, O3 and what kernels run today": all three
 * levels use per-tensor weight scales; O2 shares one dynamic activation scale
 * over the whole tensor, O3 one static scale fixed offline (values beyond the
 * calibrated range saturate).  [LLMint8] "Try it": one step = max / 127 per
 * tensor.  The per-row scale outputs below hold that one step in every entry,
 * so sq_w8a8_gemm_dequant's epilogue applies it unchanged.  These calls take
 * rows up to 40960 elements (bf16) / 25600 (fp32) (else SQ_ERR_UNSUPPORTED).
 *
 * sq_norm_smooth_absmax -- running max over all of |y|, y the norm output of
 * sq_norm_smooth_quant_per_token (same arithmetic), into absmax[0].
 *   absmax   device [1] fp32 IN/OUT (the caller starts it at zero; a running
 *            max over calls).  O2: the tensor itself; O3: the calibration
 *            tokens through the folded norm, once, offline.
 * Errors: those of sq_norm_smooth_quant_per_token.
 */
sq_status sq_norm_smooth_absmax(const void* x, sq_dtype dtype, int64_t M, int64_t K, int64_t ldx,
                                sq_norm norm, const float* gamma_folded,
                                const float* beta_folded, float eps, float* absmax,
                                void* stream);

/*
 * sq_norm_smooth_quant_per_tensor -- the norm output quantised with one step,
 * step = fl32(absmax[0] / 127); Xq = clamp(rne(fl32(y / step)), -127, 127)
 * (0 where the step is 0); x_scale[m] = step for every row.
 *   absmax   device [1] fp32 IN: max |y| (sq_norm_smooth_absmax)
 *   Xq, x_scale as for sq_norm_smooth_quant_per_token
 * Errors: those of sq_norm_smooth_quant_per_token.
 */
sq_status sq_norm_smooth_quant_per_tensor(const void* x, sq_dtype dtype, int64_t M, int64_t K,
                                          int64_t ldx, sq_norm norm, const float* gamma_folded,
                                          const float* beta_folded, float eps,
                                          const float* absmax, int8_t* Xq, float* x_scale,
                                          void* stream);

/*
 * sq_quant_per_token_given_absmax -- per-token quantisation of rows whose
 * maxima are already known (no norm): step_m = fl32(row_absmax[m] / 127),
 * Xq[m, k] = clamp(rne(fl32(x[m, k] / step_m)), -127, 127) (0 where the step
 * is 0).  With row_absmax[m] = max_k |x[m, k]| (sq_w8a8_gemm_dequant_rowmax)
 * the result equals sq_norm_smooth_quant_per_token with SQ_NORM_NONE and no
 * multiplier, bit for bit.
 * [SQ-depth] "Granularity": per-token scales, max / 127 per row.
 *   x          device [M, K] bf16 or fp32, row stride ldx
 *   row_absmax device [M] fp32 IN, 16-byte aligned
 *   Xq, x_scale as for sq_norm_smooth_quant_per_token
 * Rows up to 40960 elements (bf16) / 25600 (fp32), else SQ_ERR_UNSUPPORTED.
 * Errors: those of sq_norm_smooth_quant_per_token.
 */
sq_status sq_quant_per_token_given_absmax(const void* x, sq_dtype dtype, int64_t M, int64_t K,
                                          int64_t ldx, const float* row_absmax, int8_t* Xq,
                                          float* x_scale, void* stream);

/*
 * The row split of a Linear over several GPUs (each GPU holds a slice of the
 * input channels of x and of W; [SQ-depth] "Where the scales go in a decoder
 * block": o_proj / down_proj read unsmoothed inputs, still quantised per
 * token).  The per-token step must be the whole row's, and the accumulator
 * the whole sum, so the slices meet twice, both times exactly:
 *   1. sq_row_absmax on the local slice; all-reduce MAX of the [M] maxima;
 *   2. sq_quant_per_token_given_absmax with the reduced maxima (the step and
 *      the codes are those of the unsplit row), then sq_w8a8_gemm_dequant
 *      with SQ_EPI_I32_RAW on the local slice; all-reduce SUM of the [M, N]
 *      INT32 partial sums (integer addition: the unsplit accumulator);
 *   3. sq_dequant_i32: the epilogue of the summed accumulator.
 * The weights are quantised the same way once: the row maxima of the local
 * [N, K_slice] slice, all-reduce MAX, sq_quant_per_token_given_absmax.
 * The result is bit-identical to the unsplit call.
 *
 * sq_row_absmax -- row_absmax[m] = max_k |x[m, k]| (no norm).
 *   x          device [M, K] bf16 or fp32, row stride ldx
 *   row_absmax device [M] fp32 OUT, 16-byte aligned
 * Rows as for sq_quant_per_token_given_absmax.
 * Errors: SQ_ERR_INVALID_ARG, SQ_ERR_ALIGNMENT, SQ_ERR_UNSUPPORTED, SQ_ERR_CUDA.
 */
sq_status sq_row_absmax(const void* x, sq_dtype dtype, int64_t M, int64_t K, int64_t ldx,
                        float* row_absmax, void* stream);

/*
 * sq_dequant_i32 -- the GEMM's dequantising epilogue applied to an INT32
 * accumulator held in memory: out[m, n] = bf16(fl32(fl32(fl32(acc[m, n]) *
 * x_scale[m]) * w_scale[n])), ReLU before the rounding for SQ_EPI_BF16_RELU.
 * [SQ-depth] "Granularity": both scales applied to the INT32 accumulator.
 *   acc        device [M, N] int32, row stride lda (>= N)
 *   x_scale    device [M] fp32; w_scale device [N] fp32
 *   epi        SQ_EPI_BF16 or SQ_EPI_BF16_RELU
 *   out        device [M, N] bf16, row stride ldo (>= N)
 * Errors: SQ_ERR_INVALID_ARG (sizes, strides, null pointers, other
 *         epilogues), SQ_ERR_ALIGNMENT (acc not 4-byte, out not 2-byte
 *         aligned), SQ_ERR_CUDA.
 */
sq_status sq_dequant_i32(const int32_t* acc, int64_t M, int64_t N, int64_t lda,
                         const float* x_scale, const float* w_scale, sq_epilogue epi, void* out,
                         int64_t ldo, void* stream);

/*
 * LLM.int8()'s mixed-precision decomposition, a comparator of the smoothed
 * W8A8 layer on the same inputs.
 * [LLMint8] "Fix 1: give the outliers their own lane (LLM.int8())", "going
 * deeper -- LLM.int8() decomposition": the outlier channels
 * O = { j : max_t |X[t, j]| >= tau } (tau = 6 in the paper) go through a
 * 16-bit product, the other channels through INT8 with one absmax scale per
 * token row and one per output channel, and the two results are added.  The
 * layer is five calls:
 *   1. col_absmax [K] = max_t |X[t, j]|: sq_weight_column_max with x as its
 *      one "weight" (or sq_calibrate_absmax, SQ_NORM_NONE, into zeros);
 *   2. sq_llmint8_outliers: mask (0 on O, 1 elsewhere) and the channels of O;
 *   3. sq_norm_smooth_quant_per_token (SQ_NORM_NONE, multiplier = mask): the
 *      other channels' per-token codes (O's codes are 0 and do not set the
 *      step);
 *   4. sq_w8a8_gemm_dequant with SQ_EPI_I32_RAW and W quantised per output
 *      channel (sq_smooth_quantize_weights with s = NULL);
 *   5. sq_llmint8_combine.
 *
 * sq_llmint8_outliers -- mask[j] = col_absmax[j] >= tau ? 0 : 1; idx[0 ..
 * count) = the channels j with col_absmax[j] >= tau, ascending; *count their
 * number.
 *   col_absmax device [K] fp32 IN;  mask device [K] fp32 OUT
 *   idx        device [K] int32 OUT;  count device [1] int32 OUT
 *   tau        >= 0
 * K up to SQ_LLMINT8_MAX_K.  Pointers 4-byte aligned.
 * Errors: SQ_ERR_INVALID_ARG, SQ_ERR_ALIGNMENT, SQ_ERR_CUDA.
 */
#define SQ_LLMINT8_MAX_K 1048576

sq_status sq_llmint8_outliers(const float* col_absmax, int64_t K, float tau, float* mask,
                              int32_t* idx, int32_t* count, void* stream);

/*
 * sq_llmint8_combine -- out[m, n] = bf16(y), y = fl32(y8 + y16) (ReLU on y
 * for SQ_EPI_BF16_RELU), where
 *   y8  = fl32(fl32(fl32(acc[m, n]) * x_scale[m]) * w_scale[n]), the INT8
 *         lane dequantised as the GEMM epilogue does;
 *   y16 = fl32(s), s = the sum over the channels idx[0 .. *count), in that
 *         order, of x[m, j] * W[n, j] in fp64 (each product is exact in
 *         fp64: the 16-bit lane on the unquantised inputs).
 *   acc      device [M, N] int32, row stride lda (the INT8 lane, SQ_EPI_I32_RAW)
 *   x_scale  device [M] fp32 (step 3);  w_scale device [N] fp32
 *   x        device [M, K] bf16 / fp32, row stride ldx (the layer's input)
 *   W        device [N, K] bf16 / fp32, row stride ldw (the unquantised weights)
 *   idx, count  from sq_llmint8_outliers
 *   out      device [M, N] bf16, row stride ldo
 * Errors: SQ_ERR_INVALID_ARG (sizes, strides, dtypes, null pointers, other
 *         epilogues), SQ_ERR_ALIGNMENT, SQ_ERR_CUDA.
 */
sq_status sq_llmint8_combine(const int32_t* acc, int64_t M, int64_t N, int64_t lda,
                             const float* x_scale, const float* w_scale, const void* x,
                             sq_dtype x_dtype, int64_t ldx, const void* W, sq_dtype w_dtype,
                             int64_t ldw, int64_t K, const int32_t* idx, const int32_t* count,
                             sq_epilogue epi, void* out, int64_t ldo, void* stream);

/*
 * FP8 (e4m3) W8A8: the same smoothing, FP8 codes instead of INT8.
 * [LLMint8] "example . what you get": on GPUs with FP8 support, FP8 W8A8
 * took over INT8's role and the same smoothing still tames the activation
 * outliers before they are quantised; [SQ-map] "What it did NOT solve".
 * The pages give no FP8 arithmetic; this library's reading:
 *   e4m3 without infinities (largest finite 448), round to nearest even,
 *   saturating; step = fl32(max |y| / 448) per row; code =
 *   e4m3(fl32(y * fl32(1 / step))); a zero or subnormal step gives step 0 and
 *   all-zero codes.  The GEMM runs tcgen05 kind::f8f6f4 with an fp32
 *   accumulator; out = bf16(fl32(fl32(acc * x_scale[m]) * w_scale[n])).
 *
 * sq_norm_smooth_quant_per_token_fp8 -- sq_norm_smooth_quant_per_token with
 * FP8 codes: Xq8 device [M, K] e4m3 bytes OUT; x_scale device [M] fp32 OUT.
 * Rows up to 40960 (bf16) / 25600 (fp32) elements, else SQ_ERR_UNSUPPORTED.
 * Errors: those of sq_norm_smooth_quant_per_token.
 */
sq_status sq_norm_smooth_quant_per_token_fp8(const void* x, sq_dtype dtype, int64_t M, int64_t K,
                                             int64_t ldx, sq_norm norm,
                                             const float* gamma_folded, const float* beta_folded,
                                             float eps, uint8_t* Xq8, float* x_scale,
                                             void* stream);

/*
 * sq_smooth_quantize_weights_fp8 -- W-hat = fl32(W * s) per output channel in
 * FP8: Wq8 device [N, K] e4m3 bytes OUT, w_scale device [N] fp32 OUT.
 * Arguments and errors as for sq_smooth_quantize_weights (rows up to the
 * limits of sq_norm_smooth_quant_per_token_fp8).
 */
sq_status sq_smooth_quantize_weights_fp8(const void* W, sq_dtype dtype, int64_t N, int64_t K,
                                         int64_t ldw, const float* s, uint8_t* Wq8,
                                         float* w_scale, void* stream);

/*
 * sq_fp8_gemm_dequant -- e4m3 x e4m3 GEMM (fp32 accumulator in tensor memory)
 * with the dequantising epilogue fused.
 *   Xq8 device [M, K] e4m3 (stride K); Wq8 device [N, K] e4m3 (stride K)
 *   epi      SQ_EPI_BF16, SQ_EPI_BF16_RELU (out bf16 [M, N], stride ldo) or
 *            SQ_EPI_F32_RAW (out fp32 [M, N] = the accumulator)
 *   workspace device, caller-owned, 16-byte aligned, ws_bytes long, or NULL.
 *            With a workspace of at least
 *            sq_w8a8_gemm_workspace_size(M, N, K, 0) bytes the decode tiles
 *            (path 2, or automatic with M <= 128) run stream-K: a tile split
 *            between CTAs leaves fp32 partial sums there, which a fix-up
 *            kernel adds in ascending CTA order (the same order on every run
 *            on the same GPU model) before the epilogue.  With NULL every
 *            tile runs its whole K.  Nothing in it outlives the call.
 *   path_hint as for sq_w8a8_gemm_dequant (no explicit split-K).
 * The tensor cores' fp32 accumulation order is theirs: the accumulator
 * equals the exact sum of the decoded products to within the rounding of
 * the accumulation (not bit-exact with a sequential sum); a stream-K tile
 * adds one fp32 rounding per contributing CTA after the first.
 * Errors: those of sq_w8a8_gemm_dequant (K <= SQ_MAX_K as there);
 * SQ_ERR_WORKSPACE for a non-NULL workspace shorter than the plan needs.
 */
sq_status sq_fp8_gemm_dequant(const uint8_t* Xq8, const uint8_t* Wq8, const float* x_scale,
                              const float* w_scale, int64_t M, int64_t N, int64_t K,
                              sq_epilogue epi, void* out, int64_t ldo, void* workspace,
                              size_t ws_bytes, int path_hint, void* stream);

/*
 * sq_silu_mul_quant_per_token -- the down projection's input, SiLU(gate) * up,
 * computed from the merged gate/up projection's output and quantised per
 * token in the same pass (h is never written unless h_out is given).
 * [SQ-depth] "Where the scales go in a decoder block": the down_proj input is
 * SiLU(gate) times up; it has no norm in front, is not smoothed, and is
 * quantised with per-token scales.
 *   gate_up  device [M, 2I] bf16, row stride ld_gu: gate in columns [0, I),
 *            up in [I, 2I) (e.g. sq_w8a8_gemm_dequant's output for the
 *            merged projection)
 *   Xq       device [M, I] int8 OUT (stride I);  x_scale device [M] fp32 OUT
 *   h_out    device [M, I] bf16 OUT (stride ld_h) or NULL: h itself
 * Arithmetic (fp32, one IEEE rounding per step):
 *   e = exp(-g) by Cody-Waite reduction and a degree-7 Taylor polynomial, the
 *       argument clamped to [-87, 87] (a fixed operation sequence, under one
 *       ulp from the exact exponential);
 *   h = bf16(fl32(fl32(g * fl32(1 / fl32(1 + e))) * u));
 *   x_scale = fl32(max_k |h| / 127), Xq = clamp(rne(fl32(h / x_scale)), +-127)
 *   (0 where the row is all zero): sq_norm_smooth_quant_per_token of h with
 *   SQ_NORM_NONE, bit for bit.
 * I up to 28928 (two bf16 half-rows in shared memory), else SQ_ERR_UNSUPPORTED;
 * dtype must be SQ_BF16 (else SQ_ERR_UNSUPPORTED).
 * Errors: SQ_ERR_INVALID_ARG, SQ_ERR_ALIGNMENT (16-byte rows and pointers,
 *         I % 16), SQ_ERR_UNSUPPORTED, SQ_ERR_CUDA.
 */
sq_status sq_silu_mul_quant_per_token(const void* gate_up, sq_dtype dtype, int64_t M, int64_t I,
                                      int64_t ld_gu, int8_t* Xq, float* x_scale, void* h_out,
                                      int64_t ld_h, void* stream);

/*
 * sq_silu_mul_quant_per_token_fp8 -- sq_silu_mul_quant_per_token with FP8
 * (e4m3) codes: h as there, then the per-token FP8 quantisation of
 * sq_norm_smooth_quant_per_token_fp8 (step = fl32(max |h| / 448), codes
 * e4m3(fl32(h * fl32(1 / step)))).  Xq8 device [M, I] e4m3 bytes OUT.
 * Other arguments, limits and errors as for sq_silu_mul_quant_per_token.
 */
sq_status sq_silu_mul_quant_per_token_fp8(const void* gate_up, sq_dtype dtype, int64_t M,
                                          int64_t I, int64_t ld_gu, uint8_t* Xq8,
                                          float* x_scale, void* h_out, int64_t ld_h,
                                          void* stream);

/*
 * sq_smooth_quantize_weights_per_tensor -- W-hat = W diag(s) quantised with
 * one step for the whole matrix, fl32(max |W-hat| / 127).
 *   w_scale  device [N] fp32 OUT: the step in every entry
 *   w_absmax device [1] fp32 OUT: max |W-hat| (scratch the call overwrites)
 *   other arguments as for sq_smooth_quantize_weights
 * Errors: those of sq_smooth_quantize_weights, SQ_ERR_UNSUPPORTED.
 */
sq_status sq_smooth_quantize_weights_per_tensor(const void* W, sq_dtype dtype, int64_t N,
                                                int64_t K, int64_t ldw, const float* s,
                                                int8_t* Wq, float* w_scale, float* w_absmax,
                                                void* stream);

/*
 * sq_w8a8_gemm_workspace_size -- bytes of device workspace that
 * sq_w8a8_gemm_dequant needs for this shape and split factor (0 when the
 * chosen path needs none).  split_k = 0 asks for the automatic choice.
 */
size_t sq_w8a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int split_k);

/* What sq_w8a8_gemm_dequant will run for a shape (filled by sq_w8a8_gemm_plan). */
typedef struct sq_gemm_plan_info {
  int kernel;      /* 0: single-SM prefill tiles, 1: CTA-pair prefill tiles, 2: decode tiles */
  int tile_m;      /* rows of a tile on the MMA M side (tokens, or weight rows for decode) */
  int tile_n;      /* columns of a tile on the MMA N side */
  int split_k;     /* K slices per tile (1: none) */
  int stream_k;    /* 1: balanced K ranges per SM with a fix-up kernel */
  int ctas;        /* CTAs of the main kernel (persistent: at most one per SM) */
  int launches;    /* kernels the call launches */
  size_t workspace_bytes;
} sq_gemm_plan_info;

/*
 * sq_w8a8_gemm_plan -- host-only: the plan sq_w8a8_gemm_dequant would choose
 * for these arguments on the current device (no launch, no allocation).
 * Errors: SQ_ERR_INVALID_ARG (negative sizes, K <= 0, bad hint or split,
 * null info), SQ_ERR_UNSUPPORTED (a split on a prefill path).
 */
sq_status sq_w8a8_gemm_plan(int64_t M, int64_t N, int64_t K, int path_hint, int split_k,
                            sq_gemm_plan_info* info);

/*
 * sq_w8a8_gemm_dequant -- INT8 x INT8 -> INT32 GEMM with the dequantising
 * epilogue fused.
 * [SQ-depth] "Granularity": the GEMM computes an INT32 accumulator and applies
 * both scales in its epilogue, out = acc x scale_token[i] x scale_channel[j],
 * before converting to BF16; "The problem SmoothQuant solves": both operands
 * are 8-bit integers accumulated in INT32.
 *   Xq       device [M, K] int8 (stride K)
 *   Wq       device [N, K] int8 (stride K)
 *   x_scale  device [M] fp32;  w_scale device [N] fp32 (ignored for I32_RAW)
 *   epi      SQ_EPI_BF16, SQ_EPI_BF16_RELU (out is bf16 [M, N], stride ldo)
 *            or SQ_EPI_I32_RAW (out is int32 [M, N], stride ldo)
 *   workspace / ws_bytes  device scratch for partial sums (split-K slices,
 *            or the stream-K slots of decode tiles); at least
 *            sq_w8a8_gemm_workspace_size(M, N, K, split_k) bytes when that is
 *            non-zero, else may be NULL.  Nothing in it outlives the call, and
 *            nothing in it has to start at any value; two calls that overlap
 *            on the GPU need two workspaces.
 *   path_hint 0 = automatic, 1 = prefill tiles (tokens on the MMA M side;
 *            CTA pairs, 256-row tiles 256, 224 or 192 wide on two SMs, the width
 *            chosen to fill the SMs evenly), 2 = decode tiles (weight
 *            rows on the MMA M side, M <= 256), 3 = prefill tiles on single
 *            SMs (128 x 256)
 *   split_k  0 = automatic, else the number of K slices (decode path only;
 *            the INT32 partial sums are added exactly, so the result does not
 *            depend on it).  The automatic decode plan is stream-K: every SM
 *            runs the same number of 128-deep K steps across tile boundaries,
 *            and tiles shared by two SMs are summed by a second, small kernel
 *            (launched as a programmatic dependent of the first).
 * Accumulation is exact for K <= SQ_MAX_K (else SQ_ERR_OVERFLOW_RISK).
 * Errors: SQ_ERR_INVALID_ARG, SQ_ERR_ALIGNMENT, SQ_ERR_OVERFLOW_RISK,
 *         SQ_ERR_WORKSPACE, SQ_ERR_UNSUPPORTED, SQ_ERR_CUDA.
 */
sq_status sq_w8a8_gemm_dequant(const int8_t* Xq, const int8_t* Wq, const float* x_scale,
                               const float* w_scale, int64_t M, int64_t N, int64_t K,
                               sq_epilogue epi, void* out, int64_t ldo, void* workspace,
                               size_t ws_bytes, int path_hint, int split_k, void* stream);

/*
 * sq_w8a8_gemm_dequant_rowmax -- sq_w8a8_gemm_dequant on prefill tiles that
 * also reduces, per output row, max_n |out[m, n]| over the stored bf16 values
 * (after the ReLU for SQ_EPI_BF16_RELU).
 * [SQ-depth] "Where the scales go in a decoder block": Linears with no norm in
 * front (fc2, whose input is fc1's ReLU output) are still quantised with
 * per-token scales; each token's scale needs the maximum over the whole row,
 * which spans all of the GEMM's column tiles.  Every tile's
 * epilogue merges its rows' maxima with an atomic max, so the following
 * quantisation (sq_quant_per_token_given_absmax) reads each row once and needs
 * no reduction of its own.
 *   epi        SQ_EPI_BF16 or SQ_EPI_BF16_RELU (else SQ_ERR_INVALID_ARG)
 *   row_absmax device [M] fp32 OUT, 16-byte aligned; zeroed by the call
 *              (on the stream) before the GEMM runs
 *   path_hint  0 (= 1), 1 or 3 as for sq_w8a8_gemm_dequant; 2 (decode tiles)
 *              is SQ_ERR_INVALID_ARG
 * Other arguments as for sq_w8a8_gemm_dequant; no workspace is used.  out is
 * bit-identical to sq_w8a8_gemm_dequant's.
 * Errors: those of sq_w8a8_gemm_dequant.
 */
sq_status sq_w8a8_gemm_dequant_rowmax(const int8_t* Xq, const int8_t* Wq, const float* x_scale,
                                      const float* w_scale, int64_t M, int64_t N, int64_t K,
                                      sq_epilogue epi, void* out, int64_t ldo, float* row_absmax,
                                      int path_hint, void* stream);

/*
 * sq_linear_w8a8 -- the whole runtime layer: sq_norm_smooth_quant_per_token
 * into Xq_scratch / xscale_scratch, then sq_w8a8_gemm_dequant (automatic
 * path and split).
 *   Xq_scratch     device [M, K] int8, caller-owned
 *   xscale_scratch device [M] fp32, caller-owned
 *   workspace      as for sq_w8a8_gemm_dequant with split_k = 0
 * Errors: the union of the two calls'.
 */
sq_status sq_linear_w8a8(const void* x, sq_dtype dtype, int64_t M, int64_t K, int64_t ldx,
                         sq_norm norm, const float* gamma_folded, const float* beta_folded,
                         float eps, const int8_t* Wq, const float* w_scale, int64_t N,
                         sq_epilogue epi, void* out, int64_t ldo, int8_t* Xq_scratch,
                         float* xscale_scratch, void* workspace, size_t ws_bytes, void* stream);

/*
 * sq_w8a8_gemm_dequant_noalloc -- sq_w8a8_gemm_dequant for callers that cannot
 * allocate device memory when they call it.  (This entry point is an
 * engineering addition: the source pages have no counterpart.)
 *
 * Who needs it: code whose launch path may not allocate -- for example a
 * plugin inside an inference engine that owns all device memory, where a
 * cudaMalloc / cudaFree would also synchronise the device, or a serving loop
 * whose memory was reserved up front by a framework's allocator.
 *
 * It takes the same arguments as sq_w8a8_gemm_dequant minus the workspace.
 * The split-K partial sums go to a scratch array owned by the library: a
 * static device array of SQ_NOALLOC_SCRATCH_BYTES that every GPU which loads
 * the library keeps until the process exits.  This call allocates nothing
 * and calls no allocating routine.
 *   - Every call with M, N > 0 makes sure it knows the array's device
 *     address for the current device: the first such call on a device looks
 *     it up (with that device current), and so does the first call after the
 *     device's context was replaced (cudaDeviceReset loads the library's
 *     device code again, and the array may move).  Make that first call
 *     before any stream capture.
 *   - All calls share the one array: calls whose kernels overlap on the GPU
 *     (different streams, or different host threads) race on it.  Calls in
 *     one stream are ordered and safe.  No state carries over between calls:
 *     every partial sum is written before it is read.
 *   - With split_k = 0, a decode plan whose stream-K slots would not fit the
 *     array runs whole tiles instead (split_k = 1, no scratch).  An explicit
 *     split whose partial sums need more than SQ_NOALLOC_SCRATCH_BYTES
 *     (sq_w8a8_gemm_workspace_size tells) returns SQ_ERR_WORKSPACE and
 *     launches nothing; pass split_k = 1 (no scratch) or a smaller split.
 * Results are bit-identical to sq_w8a8_gemm_dequant's for the same plan.
 * Errors: those of sq_w8a8_gemm_dequant.
 */
#define SQ_NOALLOC_SCRATCH_BYTES (8u << 20)

sq_status sq_w8a8_gemm_dequant_noalloc(const int8_t* Xq, const int8_t* Wq,
                                       const float* x_scale, const float* w_scale, int64_t M,
                                       int64_t N, int64_t K, sq_epilogue epi, void* out,
                                       int64_t ldo, int path_hint, int split_k, void* stream);

/* Human-readable name of a status code (static storage). */
const char* sq_status_string(sq_status status);

/*
 * sq_get_device_error -- synchronises `stream`, then reads and clears the
 * device error word of the current device.  Returns SQ_OK, or the first
 * device-side error recorded since the last call (SQ_ERR_PIPELINE_TIMEOUT), or
 * SQ_ERR_CUDA if the synchronisation itself failed.
 */
sq_status sq_get_device_error(void* stream);

/*
 * sq_set_wait_limit -- diagnostics: the number of polls after which a GEMM
 * pipeline wait gives up, records SQ_ERR_PIPELINE_TIMEOUT and lets the kernel
 * drain and return (default 0 = the built-in limit of about two seconds of SM clock).
 * Affects launches made after the call, from any thread.
 */
void sq_set_wait_limit(int64_t polls);

#ifdef __cplusplus
}
#endif

#endif /* SQ_H_ */
