/*
 * w8a8.h -- C ABI of libw8a8.so, the B200 (sm_100a) SmoothQuant-style W8A8
 * linear layer: activation calibration, smoothing, SSZ weight quantization,
 * per-token activation quantization and the INT8 x INT8 -> INT32 GEMM with a
 * fused dequantization epilogue.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Matrices are row-major and contiguous.  X is [M,K] (M tokens, K input
 *    channels), W is [N,K] (N output channels; the linear-layer layout, K
 *    contiguous), Y = X W^T is [M,N].
 *  - Every pointer is caller-owned DEVICE memory (e.g. allocated by PyTorch)
 *    unless stated otherwise.  The library keeps no pointer after a call
 *    returns and allocates no device memory.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream).  Nothing synchronizes the host.  The
 *    per-token quantization kernels and the GEMMs are launched with
 *    programmatic stream serialization: they may be scheduled while the
 *    previous kernel on the stream is finishing, but wait for it to
 *    complete before reading or writing any memory, so stream order holds
 *    as for an ordinary launch.
 *  - K must be a positive multiple of 16; M and N may be 0 (nothing is done)
 *    or any positive size.  Matrix base pointers must be 16-byte aligned and
 *    vector pointers 4-byte aligned (8-byte for fp64 outputs).
 *  - Arguments are validated on the host before anything is launched; a bad
 *    argument returns an error status and leaves every output untouched.
 *    The device must be compute capability 10.0 (B200, sm_100a).
 *  - Errors are returned, never raised or aborted.  sq_last_error_detail()
 *    gives a human-readable reason for the last failure on the calling
 *    thread.
 *
 * Sources of the operations (web pages on LLM post-training quantization):
 *  [SQ]  "SmoothQuant大模型量化技术深度解析" (developer.baidu.com), section 1
 *        "SmoothQuant技术原理": s_j = max|X_j|^a / max|W_j|^(1-a), a in [0,1];
 *        activations are divided by s and weights multiplied by s, which
 *        leaves X W^T unchanged.
 *  [SSZ] "SSZ：权重量化算法说明" (msModelSlim docs), sections 算法流程,
 *        迭代优化阶段, 收敛判断, 算法参数, 使用限制: MinMax init, least-squares
 *        scale, greedy keep-if-better, relative/absolute convergence at 1e-10,
 *        at most 20 iterations, minimum scale 1e-5, int8/int4 per-channel
 *        symmetric, 2-D weights.
 *  [CQ]  CUDA INT8 quantization notes (aicoding.csdn.net), section 2.1
 *        (Q = round(R/S) + Z with calibration and saturation), section 3.2
 *        (INT8 matrix multiply), section 4.2 (dequantization fused with the
 *        integer product).
 *  [PTQ] "训练后量化（PTQ）" tutorial, "PTQ 的基本流程" (calibration pass)
 *        and "逐层量化 vs 逐通道量化" (per-channel scales).
 */
#ifndef W8A8_H
#define W8A8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SQ_OK = 0,
    SQ_ERR_NULL = 1,        /* a required pointer is NULL */
    SQ_ERR_SHAPE = 2,       /* negative size, K not a positive multiple of 16, size limit */
    SQ_ERR_DTYPE = 3,       /* dtype not supported by this entry point */
    SQ_ERR_ALIGN = 4,       /* pointer misaligned (see conventions) */
    SQ_ERR_ARG = 5,         /* scalar argument out of range (alpha, bits, max_iters) */
    SQ_ERR_UNSUPPORTED = 6, /* current device is not compute capability 10.0 */
    SQ_ERR_CUDA = 7,        /* a CUDA runtime/driver call or launch failed */
    SQ_ERR_DEVICE = 8       /* a kernel gave up on a bounded wait (see sq_device_fault) */
} sq_status;

typedef enum {
    SQ_F32 = 0,  /* IEEE binary32 */
    SQ_BF16 = 1  /* bfloat16; read exactly, written with round-to-nearest-even */
} sq_dtype;

/* Name of a status code (static string). */
const char *sq_status_string(sq_status s);

/* Reason for the last non-OK status returned on the calling host thread
 * (static thread-local buffer; "" if none). */
const char *sq_last_error_detail(void);

/* ABI version, currently 1. */
int sq_abi_version(void);

/* Reads and clears the device fault word of the current device: 0 if no
 * kernel gave up on a bounded wait since the last call, else a nonzero code
 * naming the wait.  Synchronizes `stream`.  Kernels never trap: a wait that
 * runs out of time records its code here and the kernel returns.  Codes:
 * 1 GEMM producer, 2 GEMM MMA (operands), 3 GEMM MMA (accumulator buffer),
 * 4 GEMM epilogue, 6 sq_selftest_bounded_wait, 7 W4A8 GEMM unpacking. */
sq_status sq_device_fault(void *stream, uint32_t *fault_out /* host */);

/* Debug counters (the pages' debugging advice, CUDA INT8 notes section 5:
 * copy the parameters back and compare stage by stage, in place of a
 * sanitizer).  A debug build of this library (compiled with -DW8A8_DEBUG,
 * shipped as libw8a8_debug.so) counts, in device counters, the non-finite
 * values among the input matrices the kernels read (x of sq_calib_absmax and
 * quant_act_per_token / _static / _rowsum, w of sq_smooth_fold, the smoothed
 * w of ssz_quant_weight / _asym, h of sq_layernorm_quant; each element once
 * per call) and the index checks that failed (the access is then skipped).
 * Nothing traps.  This call synchronizes `stream`, writes both totals to
 * the host and clears them; *enabled_out is 1 in a debug build.  In a
 * release build it writes zeros and *enabled_out = 0. */
sq_status sq_debug_status(void *stream, uint64_t *nonfinite_out /* host */, uint64_t *index_out /* host */,
                          int *enabled_out /* host */);

/* Test hook for the bounded waits: launches one CTA that waits, with the same
 * bounded wait the GEMM uses and a limit of limit_ms (1..10000), on an
 * mbarrier nothing ever arrives at.  The wait runs out, records fault code 6
 * in the fault word and the kernel returns; sq_device_fault() then reports 6
 * and the context stays usable.  Asynchronous on `stream`. */
sq_status sq_selftest_bounded_wait(uint32_t limit_ms, void *stream);

/* ------------------------------------------------------------------ step 1
 * Per-input-channel activation absmax calibration [SQ] max|X_j|, gathered
 * over calibration batches [PTQ]:
 *     absmax[j] = max(accumulate ? absmax[j] : 0, max_t |x[t,j]|)
 * x: [M,K] of dtype xt (SQ_F32 or SQ_BF16).  absmax: [K] fp32, in/out.
 * Exact (a max).  M == 0 with accumulate == 0 writes zeros. */
sq_status sq_calib_absmax(const void *x, sq_dtype xt, int64_t M, int64_t K,
                          float *absmax, int accumulate, void *stream);

/* ------------------------------------------------------------------ step 2
 * Smoothing factor and fold [SQ]:
 *     w_absmax[j] = max_n |w[n,j]|                       (input channel j)
 *     s[j]        = fp32( x_absmax[j]^alpha / w_absmax[j]^(1-alpha) )  (fp64 pow)
 *                   or 1 when x_absmax[j] == 0 or w_absmax[j] == 0
 *     inv_s[j]    = 1 / s[j]                              (fp32 division)
 *     w_folded[n,j] = w[n,j] * s[j]                       (fp32, optional)
 * x_absmax: [K] fp32 from sq_calib_absmax.  w: [N,K] of dtype wt.
 * alpha in [0,1].  w_absmax_out, s_out, inv_s_out: [K] fp32 outputs
 * (required).  w_folded_out: [N,K] fp32 or NULL (the fold is otherwise
 * applied on the fly by ssz_quant_weight and quant_act_per_token).
 * With w_folded_out given, s_out must be 16-byte aligned (the fold reads s
 * with 16-byte loads); SQ_ERR_ALIGN otherwise. */
sq_status sq_smooth_fold(const float *x_absmax, const void *w, sq_dtype wt,
                         int64_t N, int64_t K, float alpha, float *w_absmax_out,
                         float *s_out, float *inv_s_out, float *w_folded_out,
                         void *stream);

/* The smoothing factor alone, from both abs-max vectors [SQ]: s and inv_s
 * exactly as sq_smooth_fold computes them, with w_absmax [K] fp32 given
 * (sq_calib_absmax of w [N,K] is its w_absmax_out).  Splitting step 2 this
 * way lets the column abs-max of W run on another stream, beside the
 * activation calibration of step 1.  K a positive multiple of 16; alpha in
 * [0,1]. */
sq_status sq_smooth_factor(const float *x_absmax, const float *w_absmax, int64_t K, float alpha,
                           float *s_out, float *inv_s_out, void *stream);

/* ------------------------------------------------------------------ step 3
 * Per-output-channel symmetric weight quantization with the SSZ scale search
 * [SSZ].  For each output channel n, with w'[k] = w[n,k] * s[k] (s NULL: no
 * fold), qmax = 2^(bits-1) - 1 and Q(v, c) = clamp(rint(v / c), -qmax, qmax):
 *     scale = max(max_k |w'[k]| / qmax, 1e-5)                     (MinMax)
 *     repeat up to max_iters rounds while not converged:
 *         c  = max(sum w'Q(w',scale) / sum Q(w',scale)^2, 1e-5)   (least squares)
 *         e(c) = mean_k (w'[k] - c Q(w'[k],c))^2                  (fp64)
 *         converged = e(scale)==0 or d/e(scale) < 1e-10 or |d| < 1e-10,
 *                     d = e(scale) - e(c)
 *         keep c if e(c) < e(scale)
 *     q_out[n,:] = Q(w', scale), scale_out[n] = scale
 * bits: 8 or 4 (int4 codes are stored one per int8 byte, range [-7,7]).
 * max_iters: 0..255 (the pages use 20).  w: [N,K] of dtype wt.
 * q_out: [N,K] int8.  scale_out: [N] fp32.  mse_out: [N] fp64 or NULL
 * (final error).  iters_out: [N] int32 or NULL (rounds taken).
 * K is limited to 32768 (one channel is held on chip). */
sq_status ssz_quant_weight(const void *w, sq_dtype wt, int64_t N, int64_t K,
                           const float *s, int bits, int max_iters, int8_t *q_out,
                           float *scale_out, double *mse_out, int32_t *iters_out,
                           void *stream);

/* ------------------------------------------------------------------ step 4
 * Per-token symmetric activation quantization [CQ] 2.1 (Z = 0), with the
 * smoothing fold x' = x * inv_s (inv_s NULL: no fold):
 *     scale_out[t] = max_j |x'[t,j]| / 127
 *     q_out[t,j]   = clamp(rint(x'[t,j] / scale_out[t]), -127, 127)
 * (round half to even; an all-zero row gets scale 0 and zero codes).
 * x: [M,K] of dtype xt.  q_out: [M,K] int8.  scale_out: [M] fp32.
 * K is limited to 32768. */
sq_status quant_act_per_token(const void *x, sq_dtype xt, int64_t M, int64_t K,
                              const float *inv_s, int8_t *q_out, float *scale_out,
                              void *stream);

/* Step 4 with the row sums R[t] = sum_j q_out[t,j] (exact int32) that the
 * GEMM with asymmetric weights needs.  rowsum_out: [M] int32 or NULL (then
 * this is quant_act_per_token).  Same op, codes and scales otherwise. */
sq_status quant_act_per_token_rowsum(const void *x, sq_dtype xt, int64_t M, int64_t K,
                                     const float *inv_s, int8_t *q_out, float *scale_out,
                                     int32_t *rowsum_out, void *stream);

/* --------------------------------------------- asymmetric int8 SSZ (next)
 * [SSZ] 初始化阶段 / 迭代优化阶段 (asymmetric: scale and offset optimised
 * together by least squares); int8 only (使用限制: asymmetric int4 is not
 * supported).  Reading: w' ~ S u + m per channel, offset m in the weight
 * domain, u = clamp(rint(fl(w' - m) / S), 0, 255), stored as q = u - 128.
 *     MinMax: m = min_k w'[k], S = max((max_k w'[k] - m) / 255, 1e-5)
 *     round: least squares of w' on (u, 1) for the kept codes (fp64):
 *         den = K sum u^2 - (sum u)^2 (0: keep the pair),
 *         a = (K sum w'u - sum w' sum u) / den, b = (sum w' - a sum u) / K,
 *         candidate S = max(fp32(a), 1e-5), m = fp32(b);
 *     error, greedy keep, convergence and max_iters as ssz_quant_weight.
 * w: [N,K] of dtype wt; s: [K] fp32 fold or NULL.  q_out: [N,K] int8;
 * scale_out, offset_out: [N] fp32; mse_out [N] fp64 / iters_out [N] int32
 * or NULL.  K <= 32768, a multiple of 16. */
sq_status ssz_quant_weight_asym(const void *w, sq_dtype wt, int64_t N, int64_t K, const float *s,
                                int max_iters, int8_t *q_out, float *scale_out, float *offset_out,
                                double *mse_out, int32_t *iters_out, void *stream);

/* GEMM + dequant for asymmetric weights (scale sw, offset ow, codes
 * q = u - 128 as written by ssz_quant_weight_asym) [CQ] 3.2 / 4.2:
 *     acc[t,n] = sum_k qx[t,k] * qw[n,k]                (exact int32)
 *     A        = acc[t,n] + 128 rowsum[t]               (exact: sum qx u)
 *     y[t,n]   = yt( sx[t] * (sw[n] * (float)A + ow[n] * (float)rowsum[t]) )
 * in fp32, each product and the sum rounded once.  rowsum: [M] int32 from
 * quant_act_per_token_rowsum; ow: [N] fp32 (16-byte aligned).  Other
 * arguments as w8a8_gemm_dequant; K <= 65792 (|A| < 2^31). */
sq_status w8a8_gemm_dequant_asym(const int8_t *qx, const float *sx, const int32_t *rowsum,
                                 const int8_t *qw, const float *sw, const float *ow, int64_t M,
                                 int64_t N, int64_t K, void *y, sq_dtype yt, int32_t *acc_out,
                                 void *stream);

/* ------------------------------------------ packed int4 weights (next)
 * int4 codes (ssz_quant_weight with bits = 4, range [-7, 7]) stored two per
 * byte, and a GEMM that reads them packed: half the weight bytes.  The pages
 * have int4 per-channel SSZ but no int4 GEMM; this row is this library's.
 *
 * sq_pack_int4: packed[n, i] = (q[n,2i] & 15) | (q[n,2i+1] & 15) << 4
 * (element 2i in the low nibble, 4-bit two's complement; codes must lie in
 * [-8, 7]).  q: [N,K] int8; packed: [N, K/2] bytes; K a multiple of 32. */
sq_status sq_pack_int4(const int8_t *q, int64_t N, int64_t K, uint8_t *packed, void *stream);

/* w4a8_gemm_dequant: w8a8_gemm_dequant with the weight codes packed by
 * sq_pack_int4 (qw4: [N, K/2] bytes, 16-byte aligned).  The codes are
 * unpacked on chip; acc and y are exactly those of w8a8_gemm_dequant on
 * the unpacked codes.  K a multiple of 32, at most 131040 (the tensor
 * cores take the codes as 16 q, so the int32 accumulator holds 16 acc and
 * stays below 2^31 for any int8 qx and codes in [-8, 7]). */
sq_status w4a8_gemm_dequant(const int8_t *qx, const float *sx, const uint8_t *qw4, const float *sw,
                            int64_t M, int64_t N, int64_t K, void *y, sq_dtype yt, int32_t *acc_out,
                            void *stream);

/* -------------------------------- LayerNorm fused with step 4 (next)
 * Activation quantization fused upstream: the smoothing 1/s folded into the
 * LayerNorm that produces X ("SmoothQuant大模型量化技术深度解析" section 1: an
 * equivalent rescaling) and the quantization fused with it so that X never
 * goes to memory (CUDA INT8 notes 4.2, kernel fusion).  Per row t of
 * h [M,K] (dtype ht):
 *     mu = P(h) / K, var = P(d^2) / K, d_j = h_j - mu            (fp64)
 *     m = fp32(mu), r = fp32(1 / sqrt(var + eps))
 *     y_j = ((h_j - m) * r) * gamma_j + beta_j                   (fp32, each op rounded)
 *     x'_j = y_j * inv_s_j (fp32); codes and scale as quant_act_per_token.
 * P is the pairwise sum: the row padded with zeros to a power of two and
 * summed by recursive halving, S(lo, len) = S(lo, len/2) + S(lo + len/2,
 * len/2).  The pages fix no summation order; this tree fixes one, so the
 * statistics and the codes are reproducible bit for bit by any evaluation
 * of the same tree.
 * gamma, beta, inv_s: [K] fp32 or NULL (1, 0, 1), 16-byte aligned.  eps >= 0.
 * K: a multiple of 16 up to 16384 (one row is held in registers). */
sq_status sq_layernorm_quant(const void *h, sq_dtype ht, int64_t M, int64_t K, const float *gamma,
                             const float *beta, float eps, const float *inv_s, int8_t *q_out,
                             float *scale_out, void *stream);

/* ---------------------------------------- row-parallel (K-sharded) linear
 * The exchange of a linear whose K is split across ranks: each rank takes
 * its slice's per-token scales (quant_act_per_token), the ranks all-reduce
 * them with MAX (x -> fl(x / 127) is monotonic, so this is the unsharded
 * scale), quantize their slices at that scale, multiply (w8a8_gemm_dequant
 * with acc_out), all-reduce the int32 accumulators with SUM (exact) and
 * dequantize the sum.  The result equals the unsharded path bit for bit.
 *
 * quant_act_given_scale: q[t,j] = clamp(rint(x[t,j] * inv_s[j] / sx[t]),
 * -127, 127), 0 where sx[t] == 0 ([CQ] 2.1).  sx: [M] fp32 (device).  Shapes,
 * dtypes and alignment as quant_act_per_token (K a multiple of 16). */
sq_status quant_act_given_scale(const void *x, sq_dtype xt, int64_t M, int64_t K,
                                const float *inv_s, const float *sx, int8_t *q_out,
                                void *stream);

/* sq_dequant: y[t,n] = yt(((float)acc[t,n] * sx[t]) * sw[n]), the epilogue of
 * w8a8_gemm_dequant as its own kernel ([CQ] 4.2).  acc: [M,N] int32 and sw
 * 16-byte aligned; N a multiple of 4; y 8-byte (bf16) or 16-byte (fp32)
 * aligned. */
sq_status sq_dequant(const int32_t *acc, const float *sx, const float *sw, int64_t M, int64_t N,
                     void *y, sq_dtype yt, void *stream);

/* ------------------------------------------- static activation scale (next)
 * A per-tensor activation range calibrated offline instead of the per-token
 * scales of step 4: the moving-average abs-max of "PaddleNLP GPT
 * 量化感知训练（QAT）实战指南" section 六 (activation_quantize_type
 * moving_average_abs_max) with the range calibration and saturation of [CQ]
 * 2.1.  The pages give no moving rate; 0.9 is this library's default
 * reading (the caller passes it).
 *
 * sq_static_range_update: one calibration batch.  x_absmax: [K] fp32, that
 * batch's per-channel abs-max (sq_calib_absmax with accumulate = 0); inv_s:
 * [K] fp32 or NULL.  With a = max_j fl(x_absmax[j] * inv_s[j]) (the batch's
 * abs-max of x * inv_s):
 *     *range = first ? a : fl(fl(rate * *range) + fl(fl(1 - rate) * a))
 * range: one fp32 in device memory, in/out.  rate in [0,1]. */
sq_status sq_static_range_update(const float *x_absmax, const float *inv_s, int64_t K,
                                 float rate, int first, float *range, void *stream);

/* quant_act_static: codes at the static scale S = fl(*range / 127):
 *     q[t,j] = clamp(rint(x[t,j] * inv_s[j] / S), -127, 127)   (0 if S == 0)
 * Values beyond the range saturate.  scale_out: [M] fp32 or NULL; if given,
 * every entry receives S, so that w8a8_gemm_dequant applies the static
 * scale unchanged.  rowsum_out: [M] int32 or NULL, the exact row sums of the
 * codes (for w8a8_gemm_dequant_asym).  Shapes, dtypes and alignment as
 * quant_act_per_token. */
sq_status quant_act_static(const void *x, sq_dtype xt, int64_t M, int64_t K,
                           const float *inv_s, const float *range, int8_t *q_out,
                           float *scale_out, int32_t *rowsum_out, void *stream);

/* ------------------------------------------------------------------ step 5
 * INT8 x INT8 -> INT32 GEMM with fused per-token x per-channel dequant
 * [CQ] 3.2 and 4.2:
 *     acc[t,n] = sum_k qx[t,k] * qw[n,k]                  (exact int32)
 *     y[t,n]   = yt( ((float)acc[t,n] * sx[t]) * sw[n] )  (two fp32 multiplies)
 * qx: [M,K] int8, sx: [M] fp32, qw: [N,K] int8, sw: [N] fp32.
 * y: [M,N] of dtype yt (SQ_BF16 or SQ_F32); its row pitch must keep 16-byte
 * alignment (N % 8 == 0 for bf16, N % 4 == 0 for fp32).  acc_out: [M,N] int32
 * or NULL (the raw accumulators, for checking; needs N % 4 == 0).
 * Requires |acc| < 2^31, which holds for K <= 133144 with int8 codes. */
sq_status w8a8_gemm_dequant(const int8_t *qx, const float *sx, const int8_t *qw,
                            const float *sw, int64_t M, int64_t N, int64_t K,
                            void *y, sq_dtype yt, int32_t *acc_out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* W8A8_H */
