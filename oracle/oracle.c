/*
 * oracle.c -- plain, slow, obviously correct CPU oracle for the
 * SmoothQuant-style W8A8 linear path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  The CUDA product
 * path never links, calls or includes anything from here, and this file
 * includes nothing from the product path.
 *
 * Sources (web pages on LLM post-training quantization):
 *   [SQ]  "SmoothQuant大模型量化技术深度解析" (developer.baidu.com),
 *         section 1 "SmoothQuant技术原理": smoothing factor
 *         s_j = max|X_j|^a / max|W_j|^(1-a), activations divided by s and
 *         weights multiplied by s so the product is unchanged.
 *   [SSZ] "SSZ：权重量化算法说明" (msModelSlim docs), sections
 *         "算法流程" (MinMax init, least-squares update, greedy keep,
 *         repeat until converged or out of iterations), "迭代优化阶段"
 *         (symmetric: offset fixed at 0, only the scale is optimised),
 *         "收敛判断" (relative and absolute change tests; stop when every
 *         channel has converged), "算法参数" (20 iterations, threshold
 *         1e-10, minimum scale 1e-5), "使用限制" (int8 / int4 per-channel
 *         symmetric, 2-D weights only).
 *   [CQ]  CUDA INT8 quantization notes (aicoding.csdn.net), section 2.1
 *         "量化基础理论": Q = round(R/S) + Z with range calibration,
 *         parameter computation and saturation; section 3.2 (INT8 matrix
 *         multiply with 32-bit accumulation); section 4.2 (dequantization
 *         fused after the integer product).
 *   [PTQ] "训练后量化（PTQ）" tutorial, "PTQ 的基本流程" (calibrate on a
 *         small set, then compute scales) and "逐层量化 vs 逐通道量化"
 *         (one scale per output channel).
 *   [QAT] "PaddleNLP GPT 量化感知训练（QAT）实战指南", section 六 (the
 *         Compress configuration): activation_quantize_type
 *         'moving_average_abs_max' tracks the activation range with a
 *         moving average of the abs-max.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - channel j of W in the smoothing factor is input channel j (column j of
 *     the [N,K] weight); it is the only reading under which diag(s) cancels.
 *   - s_j = 1 when max|X_j| == 0 or max|W_j| == 0.
 *   - pow is evaluated in fp64 and rounded once to fp32.
 *   - "round" is round-half-to-even; activations clamp to [-127, 127];
 *     int4 codes clamp to [-7, 7] (qmax = 2^(bits-1) - 1).
 *   - the minimum scale floors every weight scale (init and candidates).
 *   - the quantization error is the mean over K of the squared residual,
 *     summed in fp64; a candidate's error is measured after re-quantising
 *     with the candidate scale.
 *   - the relative and absolute convergence tests are OR-ed, evaluated
 *     before the greedy update, and convergence is per channel and sticky.
 *   - the activation scale of an all-zero row is 0 and its codes are 0.
 *   - static activation scale: one per tensor, S = m / 127 with m the
 *     moving average over calibration batches of each batch's abs-max of the
 *     smoothed activations, m_1 = a_1, m_t = rate m_{t-1} + (1 - rate) a_t
 *     in fp32 (products and sum each rounded once); values beyond the range
 *     saturate to +-127.
 *
 * Arithmetic: IEEE binary32 for every quantity that decides a code, fp64
 * for error and least-squares sums, exact integers for the matrix product.
 * Build with -ffp-contract=off and without fast-math.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SSZ_CONVERGE_THRESHOLD 1e-10 /* [SSZ] 算法参数 */
#define SSZ_MIN_SCALE 1e-5f          /* [SSZ] 算法参数 */
#define ACT_QMAX 127                 /* symmetric int8, narrow range */
#define ASYM_UMAX 255                /* asymmetric int8: u in [0, 255] */

/* ---------------------------------------------------------------- step 1 */
/* Per-input-channel activation absmax, [SQ] max(|X_j|), gathered over the
 * calibration tokens ([PTQ] calibration step).  x is [M,K] row-major.
 * accumulate != 0 folds the new batch into the running max in ax. */
void oracle_calib_absmax(const float *x, int64_t M, int64_t K, float *ax,
                         int accumulate)
{
    for (int64_t j = 0; j < K; ++j)
        if (!accumulate)
            ax[j] = 0.0f;
    for (int64_t t = 0; t < M; ++t) {
        const float *row = x + t * K;
        for (int64_t j = 0; j < K; ++j) {
            float a = fabsf(row[j]);
            if (a > ax[j])
                ax[j] = a;
        }
    }
}

/* ---------------------------------------------------------------- step 2a */
/* Per-input-channel weight absmax, [SQ] max(|W_j|): w is [N,K] row-major,
 * aw[j] = max_n |w[n,j]|. */
void oracle_weight_col_absmax(const float *w, int64_t N, int64_t K, float *aw)
{
    oracle_calib_absmax(w, N, K, aw, 0);
}

/* ---------------------------------------------------------------- step 2b */
/* Smoothing factor [SQ]: s_j = ax_j^alpha / aw_j^(1-alpha), evaluated in
 * fp64 and rounded once; inv_s_j = 1/s_j in fp32. */
void oracle_smooth_factor(const float *ax, const float *aw, int64_t K,
                          float alpha, float *s, float *inv_s)
{
    double a = (double)alpha;
    for (int64_t j = 0; j < K; ++j) {
        float sj;
        if (ax[j] == 0.0f || aw[j] == 0.0f)
            sj = 1.0f;
        else
            sj = (float)(pow((double)ax[j], a) / pow((double)aw[j], 1.0 - a));
        s[j] = sj;
        inv_s[j] = 1.0f / sj;
    }
}

/* ---------------------------------------------------------------- step 2c */
/* Fold [SQ]: every column j of a [R,K] matrix times f[j] (one fp32 multiply).
 * With f = s this is W' = W diag(s); with f = 1/s it is X' = X diag(s)^-1. */
void oracle_scale_columns(const float *a, int64_t R, int64_t K, const float *f,
                          float *out)
{
    for (int64_t r = 0; r < R; ++r)
        for (int64_t j = 0; j < K; ++j)
            out[r * K + j] = a[r * K + j] * f[j];
}

/* ---------------------------------------------------------------- step 3 */
/* Symmetric code [CQ] 2.1 with Z = 0: clamp(round(w / s), -qmax, qmax),
 * fp32 division, ties to even. */
static float sym_code(float w, float s, int qmax)
{
    float r = rintf(w / s);
    if (r > (float)qmax)
        r = (float)qmax;
    if (r < -(float)qmax)
        r = -(float)qmax;
    return r;
}

/* Quantization error of one channel at scale s: mean over K of
 * (w_k - s*Q(w_k,s))^2, accumulated in fp64 in index order. */
static double channel_mse(const float *w, int64_t K, float s, int qmax)
{
    double acc = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double e = (double)w[k] - (double)s * (double)sym_code(w[k], s, qmax);
        acc += e * e;
    }
    return acc / (double)K;
}

/* SSZ scale search for one output channel ([SSZ] 算法流程, 迭代优化阶段,
 * 收敛判断), symmetric per-channel.  Returns the number of least-squares
 * rounds taken.  trace (nullable) gets the best error after the MinMax init
 * (trace[0]) and after each round (trace[1..max_iters]); unused rounds
 * repeat the final value. */
static int ssz_channel(const float *w, int64_t K, int qmax, int max_iters,
                       float *scale, double *mse, double *trace)
{
    /* MinMax observer, symmetric: scale = max|w| / qmax, offset 0. */
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(w[k]);
        if (a > amax)
            amax = a;
    }
    float s_best = amax / (float)qmax;
    if (s_best < SSZ_MIN_SCALE)
        s_best = SSZ_MIN_SCALE;
    double m_best = channel_mse(w, K, s_best, qmax);
    if (trace)
        trace[0] = m_best;

    int it = 0;
    int done = 0;
    while (it < max_iters && !done) {
        ++it;
        /* Least squares for the codes of the current best scale:
         * argmin_s sum (w - s q)^2 = sum(w q) / sum(q q). */
        double num = 0.0;
        int64_t den = 0;
        for (int64_t k = 0; k < K; ++k) {
            float q = sym_code(w[k], s_best, qmax);
            num += (double)w[k] * (double)q;
            den += (int64_t)q * (int64_t)q;
        }
        float s_cand = s_best;
        if (den != 0) {
            s_cand = (float)(num / (double)den);
            if (s_cand < SSZ_MIN_SCALE)
                s_cand = SSZ_MIN_SCALE;
        }
        double m_cand = channel_mse(w, K, s_cand, qmax);
        /* Convergence: relative OR absolute change below the threshold,
         * measured before the greedy update. */
        double delta = m_best - m_cand;
        done = (m_best == 0.0) || (delta / m_best < SSZ_CONVERGE_THRESHOLD) ||
               (fabs(delta) < SSZ_CONVERGE_THRESHOLD);
        /* Greedy: keep the candidate only if it lowers the error. */
        if (m_cand < m_best) {
            s_best = s_cand;
            m_best = m_cand;
        }
        if (trace)
            trace[it] = m_best;
    }
    if (trace)
        for (int r = it + 1; r <= max_iters; ++r)
            trace[r] = m_best;
    *scale = s_best;
    *mse = m_best;
    return it;
}

/* Per-output-channel symmetric weight quantization with the SSZ search.
 * w is the already-smoothed [N,K] fp32 weight.  bits is 8 or 4.
 * Outputs: codes q [N,K] (int4 codes stored one per byte), scale [N],
 * mse [N] (nullable), iters [N] (nullable), trace [N, max_iters+1]
 * (nullable).  Returns 0, or -1 on an argument the pages do not support. */
int oracle_ssz_quant_weight(const float *w, int64_t N, int64_t K, int bits,
                            int max_iters, int8_t *q, float *scale,
                            double *mse, int32_t *iters, double *trace)
{
    if (bits != 8 && bits != 4)
        return -1; /* [SSZ] 使用限制: int8 and int4 only */
    if (N < 0 || K <= 0 || max_iters < 0)
        return -1;
    int qmax = (1 << (bits - 1)) - 1;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < N; ++n) {
        const float *row = w + n * K;
        float s;
        double m;
        int it = ssz_channel(row, K, qmax, max_iters, &s, &m,
                             trace ? trace + n * (int64_t)(max_iters + 1) : 0);
        scale[n] = s;
        if (mse)
            mse[n] = m;
        if (iters)
            iters[n] = it;
        for (int64_t k = 0; k < K; ++k)
            q[n * K + k] = (int8_t)sym_code(row[k], s, qmax);
    }
    return 0;
}

/* Codes of a [N,K] weight at given per-row scales (stage-wise parity: the
 * codes a scale implies). */
void oracle_weight_codes(const float *w, int64_t N, int64_t K, int bits,
                         const float *scale, int8_t *q)
{
    int qmax = (1 << (bits - 1)) - 1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            q[n * K + k] = (int8_t)sym_code(w[n * K + k], scale[n], qmax);
}

/* The error of one channel at a given scale (exposed for the pins). */
double oracle_channel_mse(const float *w, int64_t K, float s, int bits)
{
    return channel_mse(w, K, s, (1 << (bits - 1)) - 1);
}

/* ------------------------------------------------- asymmetric int8 SSZ */
/* Asymmetric code ([SSZ] 迭代优化阶段, 非对称量化: scale and offset both
 * free; [CQ] 2.1 Q = round(R/S) + Z).  Reading: the offset m lives in the
 * weight domain, w ~ S u + m with u = clamp(rint(fl(w - m) / S), 0, 255)
 * (all 256 levels of int8; stored as q = u - 128). */
static float asym_code(float w, float S, float m)
{
    float v = w - m;
    float r = rintf(v / S);
    if (r > (float)ASYM_UMAX)
        r = (float)ASYM_UMAX;
    if (r < 0.0f)
        r = 0.0f;
    return r;
}

/* mean over K of (w - (S u + m))^2 in fp64, index order, re-quantising at
 * (S, m). */
static double channel_mse_asym(const float *w, int64_t K, float S, float m)
{
    double acc = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double u = (double)asym_code(w[k], S, m);
        double e = (double)w[k] - ((double)S * u + (double)m);
        acc += e * e;
    }
    return acc / (double)K;
}

/* One channel: MinMax init (m = min w, S = (max w - min w) / 255, floored),
 * then rounds of least squares for (S, m) given the codes of the kept pair,
 *     den = K sum u^2 - (sum u)^2,  a = (K sum wu - sum w sum u) / den,
 *     b = (sum w - a sum u) / K   (fp64; den == 0 keeps the pair),
 * candidate S = max(fp32(a), 1e-5), m = fp32(b); the error, greedy keep and
 * convergence tests are those of the symmetric search. */
static int ssz_channel_asym(const float *w, int64_t K, int max_iters, float *scale, float *offset,
                            double *mse, double *trace)
{
    float wmin = w[0], wmax = w[0];
    for (int64_t k = 1; k < K; ++k) {
        if (w[k] < wmin)
            wmin = w[k];
        if (w[k] > wmax)
            wmax = w[k];
    }
    float s_best = (wmax - wmin) / (float)ASYM_UMAX;
    if (s_best < SSZ_MIN_SCALE)
        s_best = SSZ_MIN_SCALE;
    float m_off = wmin;
    double e_best = channel_mse_asym(w, K, s_best, m_off);
    if (trace)
        trace[0] = e_best;
    int it = 0;
    int done = 0;
    while (it < max_iters && !done) {
        ++it;
        double sw = 0.0, swu = 0.0;
        int64_t su = 0, suu = 0;
        for (int64_t k = 0; k < K; ++k) {
            float u = asym_code(w[k], s_best, m_off);
            sw += (double)w[k];
            swu += (double)w[k] * (double)u;
            su += (int64_t)u;
            suu += (int64_t)u * (int64_t)u;
        }
        double den = (double)K * (double)suu - (double)su * (double)su;
        float s_cand = s_best, m_cand = m_off;
        if (den != 0.0) {
            double a = ((double)K * swu - sw * (double)su) / den;
            double b = (sw - a * (double)su) / (double)K;
            s_cand = (float)a;
            if (s_cand < SSZ_MIN_SCALE)
                s_cand = SSZ_MIN_SCALE;
            m_cand = (float)b;
        }
        double e_cand = channel_mse_asym(w, K, s_cand, m_cand);
        double delta = e_best - e_cand;
        done = (e_best == 0.0) || (delta / e_best < SSZ_CONVERGE_THRESHOLD) ||
               (fabs(delta) < SSZ_CONVERGE_THRESHOLD);
        if (e_cand < e_best) {
            s_best = s_cand;
            m_off = m_cand;
            e_best = e_cand;
        }
        if (trace)
            trace[it] = e_best;
    }
    if (trace)
        for (int r = it + 1; r <= max_iters; ++r)
            trace[r] = e_best;
    *scale = s_best;
    *offset = m_off;
    *mse = e_best;
    return it;
}

/* Per-output-channel asymmetric int8 weight quantization with the SSZ
 * search (int4 asymmetric is unsupported on the SSZ page, 使用限制).
 * w: smoothed [N,K] fp32.  Outputs: q [N,K] int8 = u - 128, scale [N],
 * offset [N] (weight domain), mse/iters/trace nullable as in the symmetric
 * search.  Returns 0, or -1 on a bad argument. */
int oracle_ssz_quant_weight_asym(const float *w, int64_t N, int64_t K, int max_iters, int8_t *q,
                                 float *scale, float *offset, double *mse, int32_t *iters,
                                 double *trace)
{
    if (N < 0 || K <= 0 || max_iters < 0)
        return -1;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < N; ++n) {
        const float *row = w + n * K;
        float S, m;
        double e;
        int it = ssz_channel_asym(row, K, max_iters, &S, &m, &e,
                                  trace ? trace + n * (int64_t)(max_iters + 1) : 0);
        scale[n] = S;
        offset[n] = m;
        if (mse)
            mse[n] = e;
        if (iters)
            iters[n] = it;
        for (int64_t k = 0; k < K; ++k)
            q[n * K + k] = (int8_t)((int)asym_code(row[k], S, m) - 128);
    }
    return 0;
}

/* Codes of a [N,K] weight at given per-row (S, m) (stage-wise parity: the
 * stored codes q = u - 128 a scale and offset imply, [SSZ] 迭代优化阶段). */
void oracle_weight_codes_asym(const float *w, int64_t N, int64_t K, const float *S,
                              const float *m, int8_t *q)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            q[n * K + k] = (int8_t)((int)asym_code(w[n * K + k], S[n], m[n]) - 128);
}

/* The error of one channel at a given (S, m) (exposed for the pins). */
double oracle_channel_mse_asym(const float *w, int64_t K, float S, float m)
{
    return channel_mse_asym(w, K, S, m);
}

/* ---------------------------------------------------------------- step 4 */
/* Per-token symmetric activation quantization ([CQ] 2.1, Z = 0): with
 * x' = x * inv_s (inv_s nullable: no smoothing), sx_t = max_j|x'_tj| / 127
 * and q_tj = clamp(rint(x'_tj / sx_t), -127, 127); an all-zero row gives
 * sx_t = 0 and zero codes. */
void oracle_quant_act_per_token(const float *x, int64_t M, int64_t K,
                                const float *inv_s, int8_t *q, float *sx)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < M; ++t) {
        const float *row = x + t * K;
        float amax = 0.0f;
        for (int64_t j = 0; j < K; ++j) {
            float v = inv_s ? row[j] * inv_s[j] : row[j];
            float a = fabsf(v);
            if (a > amax)
                amax = a;
        }
        float s = amax / (float)ACT_QMAX;
        sx[t] = s;
        for (int64_t j = 0; j < K; ++j) {
            float v = inv_s ? row[j] * inv_s[j] : row[j];
            q[t * K + j] = (s == 0.0f) ? (int8_t)0 : (int8_t)sym_code(v, s, ACT_QMAX);
        }
    }
}

/* ------------------------------------------- LayerNorm fused with step 4 */
/* Pairwise (recursive halving) fp64 sum of v[0..K-1] padded with zeros to a
 * power of two P >= K: S(lo, len) = S(lo, len/2) + S(lo + len/2, len/2),
 * S(i, 1) = v[i] (0 past K).  The order is fixed by the definition, not by
 * an implementation, so any evaluation of this tree gives the same bits
 * (zero subtrees add exactly 0; padding to a larger power of two changes at
 * most the sign of a zero sum). */
static double pairwise(const double *v, int64_t K, int64_t lo, int64_t len)
{
    if (lo >= K)
        return 0.0;
    if (len == 1)
        return v[lo];
    int64_t h = len / 2;
    return pairwise(v, K, lo, h) + pairwise(v, K, lo + h, h);
}

double oracle_pairwise_sum(const double *v, int64_t K)
{
    int64_t P = 1;
    while (P < K)
        P *= 2;
    return K > 0 ? pairwise(v, K, 0, P) : 0.0;
}

/* Activation quantization fused upstream: the smoothing 1/s folded into the
 * LayerNorm that produces X (SmoothQuant page, section 1: the scaling is an
 * equivalent transform; CUDA INT8 notes 4.2: fuse quantization with the
 * neighbouring op so the intermediate never goes to memory).  Per row t of
 * h [M,K]:
 *     mu  = P(h) / K,  var = P(d^2) / K,  d_j = h_j - mu         (fp64)
 *     m = fp32(mu), r = fp32(1 / sqrt(var + eps))
 * with P the pairwise sum above (the pages fix no summation order; a fixed
 * tree makes the statistics, and hence the codes, reproducible bit for bit);
 *     y_j = ((h_j - m) * r) * gamma_j + beta_j                  (fp32, each op rounded)
 *     x'_j = y_j * inv_s_j (fp32), then the per-token codes and scale of step 4.
 * gamma, beta, inv_s nullable (1, 0, 1).  Also writes y (the LayerNorm
 * output, nullable) and stats (nullable, [M,2]: mu and var in fp64) so the
 * pins can check them. */
void oracle_layernorm_quant(const float *h, int64_t M, int64_t K, const float *gamma,
                            const float *beta, float eps, const float *inv_s, int8_t *q,
                            float *sx, float *y_out, double *stats)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < M; ++t) {
        const float *row = h + t * K;
        double *tmp = (double *)malloc((size_t)K * sizeof(double));
        for (int64_t j = 0; j < K; ++j)
            tmp[j] = (double)row[j];
        double mu = oracle_pairwise_sum(tmp, K) / (double)K;
        for (int64_t j = 0; j < K; ++j) {
            double d = (double)row[j] - mu;
            tmp[j] = d * d;
        }
        double ss = oracle_pairwise_sum(tmp, K);
        free(tmp);
        if (stats) {
            stats[2 * t] = mu;
            stats[2 * t + 1] = ss / (double)K;
        }
        double rstd = 1.0 / sqrt(ss / (double)K + (double)eps);
        float m32 = (float)mu, r32 = (float)rstd;
        float *y = (float *)malloc((size_t)K * sizeof(float));
        float amax = 0.0f;
        for (int64_t j = 0; j < K; ++j) {
            float g = gamma ? gamma[j] : 1.0f;
            float b = beta ? beta[j] : 0.0f;
            float n = (row[j] - m32) * r32;
            float yj = n * g + b;
            if (y_out)
                y_out[t * K + j] = yj;
            float v = inv_s ? yj * inv_s[j] : yj;
            y[j] = v;
            float a = fabsf(v);
            if (a > amax)
                amax = a;
        }
        float s = amax / (float)ACT_QMAX;
        sx[t] = s;
        for (int64_t j = 0; j < K; ++j)
            q[t * K + j] = (s == 0.0f) ? (int8_t)0 : (int8_t)sym_code(y[j], s, ACT_QMAX);
        free(y);
    }
}

/* ---------------------------------------- row-parallel (K-sharded) linear */
/* Codes of x' = x * inv_s at given per-row scales sx[t] (sx[t] == 0: zero
 * codes).  With K split across ranks, each rank's per-token scale is
 * fl(max_local / 127); the MAX over ranks of those equals the unsharded
 * scale (x -> fl(x / 127) is monotonic), and every rank then quantizes its
 * slice at that scale ([CQ] 2.1), so the codes are the unsharded codes. */
void oracle_quant_act_given_scale(const float *x, int64_t M, int64_t K, const float *inv_s,
                                  const float *sx, int8_t *q)
{
    for (int64_t t = 0; t < M; ++t)
        for (int64_t j = 0; j < K; ++j) {
            float v = inv_s ? x[t * K + j] * inv_s[j] : x[t * K + j];
            q[t * K + j] = (sx[t] == 0.0f) ? (int8_t)0 : (int8_t)sym_code(v, sx[t], ACT_QMAX);
        }
}

/* ------------------------------------------------- static activation scale */
/* Abs-max of the smoothed activations x' = x * inv_s over one calibration
 * batch x [M,K] (inv_s nullable): the per-tensor range [CQ] 2.1 "范围校准". */
float oracle_static_batch_absmax(const float *x, int64_t M, int64_t K, const float *inv_s)
{
    float amax = 0.0f;
    for (int64_t t = 0; t < M; ++t)
        for (int64_t j = 0; j < K; ++j) {
            float v = inv_s ? x[t * K + j] * inv_s[j] : x[t * K + j];
            float a = fabsf(v);
            if (a > amax)
                amax = a;
        }
    return amax;
}

/* Moving average of the per-batch abs-max ([QAT] moving_average_abs_max;
 * [CQ] 2.1: a moving average of the range is more robust than raw min/max):
 * the first batch sets the state, later ones blend in with weight 1 - rate. */
float oracle_static_ema(float state, float a, float rate, int first)
{
    if (first)
        return a;
    float keep = rate * state;
    float w = 1.0f - rate;
    float add = w * a;
    return keep + add;
}

/* Static per-tensor activation quantization ([CQ] 2.1 with Z = 0, one scale
 * for the whole tensor): S = m / 127, q = clamp(rint(x' / S), -127, 127);
 * S == 0 gives zero codes. */
void oracle_quant_act_static(const float *x, int64_t M, int64_t K, const float *inv_s, float m,
                             int8_t *q)
{
    float S = m / (float)ACT_QMAX;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < M; ++t)
        for (int64_t j = 0; j < K; ++j) {
            float v = inv_s ? x[t * K + j] * inv_s[j] : x[t * K + j];
            q[t * K + j] = (S == 0.0f) ? (int8_t)0 : (int8_t)sym_code(v, S, ACT_QMAX);
        }
}

/* ---------------------------------------------------------------- step 5 */
/* Exact integer product [CQ] 3.2: acc[t,n] = sum_k qx[t,k] * qw[n,k], both
 * operands K-contiguous (the weight in [N,K] linear-layer layout).  The sum
 * is taken in int64; |acc| <= K * 127^2 < 2^31 for K < 133144. */
void oracle_gemm_i8(const int8_t *qx, const int8_t *qw, int64_t M, int64_t N,
                    int64_t K, int32_t *acc)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < M; ++t)
        for (int64_t n = 0; n < N; ++n) {
            int64_t sum = 0;
            for (int64_t k = 0; k < K; ++k)
                sum += (int64_t)qx[t * K + k] * (int64_t)qw[n * K + k];
            acc[t * N + n] = (int32_t)sum;
        }
}

/* fp32 -> bf16 with round-to-nearest-even; NaN maps to a quiet NaN. */
static uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u)
        return (uint16_t)((u >> 16) | 0x0040u);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* Dequantization [CQ] 4.2: y[t,n] = ((float)acc[t,n] * sx[t]) * sw[n], two
 * fp32 multiplies in that order.  y_f32 and y_bf16 are each nullable. */
void oracle_dequant(const int32_t *acc, const float *sx, const float *sw,
                    int64_t M, int64_t N, float *y_f32, uint16_t *y_bf16)
{
    for (int64_t t = 0; t < M; ++t)
        for (int64_t n = 0; n < N; ++n) {
            float y = ((float)acc[t * N + n] * sx[t]) * sw[n];
            if (y_f32)
                y_f32[t * N + n] = y;
            if (y_bf16)
                y_bf16[t * N + n] = f32_to_bf16_rne(y);
        }
}

/* ------------------------------------------------------- packed int4 */
/* Two int4 codes per byte (the pages print no packed layout, so this one is
 * a reading; the int4 codes themselves are the int4 per-channel symmetric
 * case of "SSZ：权重量化算法说明", 使用限制).
 * Reading: element 2i in the low nibble, 2i+1 in the high nibble, each in
 * 4-bit two's complement; codes must lie in [-8, 7].  K is even. */
void oracle_pack_int4(const int8_t *q, int64_t N, int64_t K, uint8_t *packed)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t i = 0; i < K / 2; ++i) {
            unsigned lo = (unsigned)(q[n * K + 2 * i] & 0x0F);
            unsigned hi = (unsigned)(q[n * K + 2 * i + 1] & 0x0F);
            packed[n * (K / 2) + i] = (uint8_t)(lo | (hi << 4));
        }
}

/* The inverse: sign-extend each nibble back to an int8 code. */
void oracle_unpack_int4(const uint8_t *packed, int64_t N, int64_t K, int8_t *q)
{
    for (int64_t n = 0; n < N; ++n)
        for (int64_t i = 0; i < K / 2; ++i) {
            int b = packed[n * (K / 2) + i];
            int lo = b & 0x0F, hi = (b >> 4) & 0x0F;
            q[n * K + 2 * i] = (int8_t)(lo >= 8 ? lo - 16 : lo);
            q[n * K + 2 * i + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
        }
}

/* Row sums R_t = sum_k qx[t,k] of the activation codes (exact). */
void oracle_act_rowsum(const int8_t *qx, int64_t M, int64_t K, int32_t *R)
{
    for (int64_t t = 0; t < M; ++t) {
        int64_t r = 0;
        for (int64_t k = 0; k < K; ++k)
            r += qx[t * K + k];
        R[t] = (int32_t)r;
    }
}

/* Dequant with asymmetric weights ([CQ] 4.2 with the zero point of 2.1):
 * w ~ S_n u + m_n with u = q + 128, so
 *     sum_k sx_t qx[t,k] (S_n u[n,k] + m_n) = sx_t (S_n A + m_n R_t),
 *     A = acc[t,n] + 128 R_t  (exact int32; acc = sum qx q of the stored codes)
 * in fp32: y = fl(sx_t * fl(fl(S_n * (float)A) + fl(m_n * (float)R_t))). */
void oracle_dequant_asym(const int32_t *acc, const int32_t *R, const float *sx, const float *S,
                         const float *m, int64_t M, int64_t N, float *y_f32, uint16_t *y_bf16)
{
    for (int64_t t = 0; t < M; ++t)
        for (int64_t n = 0; n < N; ++n) {
            int32_t A = acc[t * N + n] + 128 * R[t];
            float p = S[n] * (float)A;
            float o = m[n] * (float)R[t];
            float y = sx[t] * (p + o);
            if (y_f32)
                y_f32[t * N + n] = y;
            if (y_bf16)
                y_bf16[t * N + n] = f32_to_bf16_rne(y);
        }
}

/* Elementwise fp32 -> bf16 (RNE) for arrays, so callers round exactly as
 * the dequant does. */
void oracle_to_bf16(const float *a, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = f32_to_bf16_rne(a[i]);
}
