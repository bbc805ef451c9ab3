// ssz.cu -- step 3: per-output-channel symmetric weight quantization with the
// SSZ least-squares scale search.
//
// Source: "SSZ：权重量化算法说明" (msModelSlim docs):
//   算法流程 / 初始化阶段: MinMax observer gives the initial scale (symmetric:
//     scale = max|w| / qmax, offset 0);
//   迭代优化阶段: least squares gives the best scale for the current codes,
//     sum(w q) / sum(q q); greedy: keep new parameters only if the
//     quantization error improves;
//   收敛判断: relative change (best - cur)/best < threshold or absolute change
//     |best - cur| < threshold; stop when every channel has converged;
//   算法参数: 20 iterations, threshold 1e-10, minimum scale 1e-5;
//   使用限制: int8 and int4, per-channel symmetric, 2-D weights.
// The SmoothQuant fold W' = W diag(s) ("SmoothQuant大模型量化技术深度解析",
// section 1) is applied as the row is loaded.
//
// Readings (shared with the CPU oracle): the error is the mean over K of
// (w - c Q(w,c))^2 summed in fp64 after re-quantising at the candidate c;
// the relative and absolute tests are OR-ed, taken before the greedy update,
// and a channel stops for good once it meets them; the minimum scale floors
// the MinMax scale and every candidate; int4 codes are [-7, 7].
//
// Design: one CTA per output channel.  The folded row stays in registers for
// the whole search (E fp32 values per thread), so W is read from HBM once and
// the codes written once.  Each round is ONE pass over the row that computes,
// for the candidate scale c, the codes Q(w,c), the error sum (w - c q)^2, and
// the least-squares sums sum(w q), sum(q q) for the next candidate: when the
// candidate is kept, the next round's least squares needs exactly these sums;
// when it is not kept the channel has converged (d <= 0 passes the relative
// test), so no round ever needs the sums of an older scale.  The three sums
// are reduced across the CTA (warp shuffles, then the warps in a fixed order
// so every thread takes the same decisions).
#include "common.cuh"

namespace w8a8 {

// Elements per thread for 2048 < K <= W8A8_SSZ_MID_MAX_K (a build-time
// tuning choice; 32 elements per thread otherwise above 2048).
#ifndef W8A8_SSZ_MID_E
#define W8A8_SSZ_MID_E 32
#endif
#ifndef W8A8_SSZ_MID_MAX_K
#define W8A8_SSZ_MID_MAX_K 8192
#endif

constexpr double kSszThreshold = 1e-10;
constexpr float kSszMinScale = 1e-5f;

struct Sums {
    double err;   // sum (w - c q)^2
    double wq;    // sum w q
    int den;      // sum q q  (<= 32768 * 127^2 < 2^31)
};

// One pass over this thread's elements at scale c.  Per element: the code
// on the FP32 pipe (magic-constant rounding, as sym_code_i), the code widened
// to fp64 from its bits, w widened by one F2F, the residual w - c q rounded
// once (c*q is exact in fp64), and three accumulations, split four ways so
// the fp64 adds do not form one long dependency chain.  The distance of each
// scaled value to its nearest integer is folded into a running max instead
// of branching per element; if any element of this thread came within 2^-15
// of a tie, the thread redoes its sums from the shared-memory copy of its
// elements with the exact IEEE quotient where needed (rare: about one thread
// in 500 per pass).
template <int C>
__device__ __forceinline__ Sums row_pass(const float (&w)[C][8], const bool (&live)[C],
                                         const float *__restrict__ wsh, float c, float qmax) {
    const float r = __fdiv_rn(1.0f, c);  // c >= 1e-5, so r is finite
    const double cd = (double)c;
    const float lo = kRoundMagic - qmax, hi = kRoundMagic + qmax;
    double err[4] = {0.0, 0.0, 0.0, 0.0}, wq[4] = {0.0, 0.0, 0.0, 0.0};
    int den = 0;
    float dmax = 0.0f;
#pragma unroll
    for (int k = 0; k < C; ++k) {
        if (!live[k]) continue;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float y = w[k][i] * r;
            const float t = y + kRoundMagic;
            dmax = fmaxf(dmax, fabsf(y - (t - kRoundMagic)));
            const int q = __float_as_int(fminf(fmaxf(t, lo), hi)) - kRoundMagicBits;
            const double qd = code_to_f64(q);
            const double wd = (double)w[k][i];
            const double e = fma(-cd, qd, wd);
            err[i & 3] = fma(e, e, err[i & 3]);
            wq[i & 3] = fma(wd, qd, wq[i & 3]);  // w*q is exact in fp64
            den += q * q;
        }
    }
    if (dmax >= 0.5f - 3.0517578125e-05f) {
        // rare exact path, rolled over the shared-memory copy (same order)
        const int T_ = blockDim.x;
        double err_x = 0.0, wq_x = 0.0;
        den = 0;
#pragma unroll 1
        for (int k = 0; k < C; ++k) {
            if (!live[k]) continue;
            const float *p = wsh + (k * T_ + threadIdx.x) * 8;
#pragma unroll 1
            for (int i = 0; i < 8; ++i) {
                const int q = sym_code_i(p[i], c, r, qmax);
                const double qd = code_to_f64(q);
                const double wd = (double)p[i];
                const double e = fma(-cd, qd, wd);
                err_x = fma(e, e, err_x);
                wq_x = fma(wd, qd, wq_x);
                den += q * q;
            }
        }
        return {err_x, wq_x, den};
    }
    return {(err[0] + err[1]) + (err[2] + err[3]), (wq[0] + wq[1]) + (wq[2] + wq[3]), den};
}

// Block-wide sum of Sums; every thread gets the same result (warps are
// combined in index order).  `slot` alternates so one barrier per call is
// enough.
__device__ __forceinline__ Sums block_sum(Sums s, Sums (*red)[32], int slot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        s.err += __shfl_xor_sync(0xffffffffu, s.err, o);
        s.wq += __shfl_xor_sync(0xffffffffu, s.wq, o);
        s.den += __shfl_xor_sync(0xffffffffu, s.den, o);
    }
    if (lane == 0) red[slot][warp] = s;
    __syncthreads();
    Sums t = red[slot][0];
    for (int w = 1; w < nwarps; ++w) {
        t.err += red[slot][w].err;
        t.wq += red[slot][w].wq;
        t.den += red[slot][w].den;
    }
    return t;
}

template <typename T, int E, bool FOLD>
__global__ void __launch_bounds__(512)
ssz_kernel(const T *__restrict__ wg, int64_t N, int64_t K, const float *__restrict__ s, float qmax,
           int max_iters, int8_t *__restrict__ q_out, float *__restrict__ scale_out,
           double *__restrict__ mse_out, int32_t *__restrict__ iters_out) {
    constexpr int C = E / 8;
    __shared__ Sums red[2][32];
    __shared__ float redmax[32];
    extern __shared__ float wsh[];  // this channel's folded row (exact-path copy)
    const int T_ = blockDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = T_ >> 5;

    for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
        // ---- load the folded row into registers
        float w[C][8];
        bool live[C];
        float amax = 0.0f;
#pragma unroll
        for (int k = 0; k < C; ++k) {
            int64_t j = ((int64_t)k * T_ + threadIdx.x) * 8;
            live[k] = j < K;
            if (live[k]) {
                Vec8<T>::load(wg + n * K + j, w[k]);
                if (FOLD) {
                    float f[8];
                    load8_f32(s + j, f);
#pragma unroll
                    for (int i = 0; i < 8; ++i) w[k][i] = w[k][i] * f[i];
                }
                float4 *dst = reinterpret_cast<float4 *>(wsh + j);
                dst[0] = make_float4(w[k][0], w[k][1], w[k][2], w[k][3]);
                dst[1] = make_float4(w[k][4], w[k][5], w[k][6], w[k][7]);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) w[k][i] = 0.0f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(w[k][i]));
        }
        // ---- MinMax init
        amax = warp_max(amax);
        if (lane == 0) redmax[warp] = amax;
        __syncthreads();
        amax = redmax[0];
        for (int i = 1; i < nwarps; ++i) amax = fmaxf(amax, redmax[i]);

        // Round 0 evaluates the MinMax scale; round it >= 1 evaluates the
        // least-squares candidate built from the sums of the kept scale.  One
        // inlined pass serves both, which keeps the kernel small.
        const double kd = (double)K;
        float s_best = fmaxf(__fdiv_rn(amax, qmax), kSszMinScale);
        float c = s_best;
        double m_best = 0.0;
        Sums cur = {0.0, 0.0, 0};
        int it = 0;
        int slot = 0;
        for (;;) {
            const Sums nxt = block_sum(row_pass<C>(w, live, wsh, c, qmax), red, slot);
            slot ^= 1;
            const double m_c = nxt.err / kd;
            if (it == 0) {
                m_best = m_c;
                cur = nxt;
            } else {
                const double delta = m_best - m_c;
                const bool done = (m_best == 0.0) || (delta / m_best < kSszThreshold) ||
                                  (fabs(delta) < kSszThreshold);
                if (m_c < m_best) {
                    s_best = c;
                    m_best = m_c;
                    cur = nxt;
                }
                if (done) break;
            }
            if (it == max_iters) break;
            ++it;
            c = (cur.den != 0) ? fmaxf((float)(cur.wq / (double)cur.den), kSszMinScale) : s_best;
        }

        // ---- codes at the kept scale
        const float r = __fdiv_rn(1.0f, s_best);
#pragma unroll
        for (int k = 0; k < C; ++k) {
            if (!live[k]) continue;
            int code[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) code[i] = sym_code_i(w[k][i], s_best, r, qmax);
            *reinterpret_cast<uint2 *>(q_out + n * K + ((int64_t)k * T_ + threadIdx.x) * 8) =
                pack8_codes(code);
        }
        if (threadIdx.x == 0) {
            scale_out[n] = s_best;
            if (mse_out) mse_out[n] = m_best;
            if (iters_out) iters_out[n] = it;
        }
        // redmax / red slots are reused by the next row: make sure every
        // thread has read them
        __syncthreads();
    }
}

template <typename T, int E>
static void launch_ssz(const void *w, int64_t N, int64_t K, const float *s, int bits, int max_iters,
                       int8_t *q, float *scale, double *mse, int32_t *iters, int sms, cudaStream_t st) {
    const int threads = (int)ceil_div(ceil_div(K, E), 32) * 32;
    const float qmax = (float)((1 << (bits - 1)) - 1);
    const int per_sm = std::max(1, 2048 / threads);
    const int64_t grid = std::min<int64_t>(N, (int64_t)sms * per_sm * 4);
    const size_t smem = (size_t)threads * E * sizeof(float);  // <= 512 * 64 * 4 = 128 KB
    auto kern = s ? ssz_kernel<T, E, true> : ssz_kernel<T, E, false>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<(unsigned)grid, threads, smem, st>>>((const T *)w, N, K, s, qmax, max_iters, q, scale, mse, iters);
}

}  // namespace w8a8

using namespace w8a8;

extern "C" sq_status ssz_quant_weight(const void *w, sq_dtype wt, int64_t N, int64_t K, const float *s,
                                      int bits, int max_iters, int8_t *q_out, float *scale_out,
                                      double *mse_out, int32_t *iters_out, void *stream) {
    if (N > 0 && (!w || !q_out || !scale_out)) return fail(SQ_ERR_NULL, "ssz_quant_weight: NULL pointer");
    if (wt != SQ_F32 && wt != SQ_BF16) return fail(SQ_ERR_DTYPE, "ssz_quant_weight: dtype %d", (int)wt);
    if (N < 0 || K <= 0 || K % 16 != 0 || K > 32768)
        return fail(SQ_ERR_SHAPE, "ssz_quant_weight: N=%lld K=%lld (K must be a multiple of 16 in [16, 32768])",
                    (long long)N, (long long)K);
    if (bits != 8 && bits != 4)
        return fail(SQ_ERR_ARG, "ssz_quant_weight: bits=%d (int8 and int4 only)", bits);
    if (max_iters < 0 || max_iters > 255)
        return fail(SQ_ERR_ARG, "ssz_quant_weight: max_iters=%d outside [0, 255]", max_iters);
    if (N == 0) return SQ_OK;
    if (!aligned(w, 16) || !aligned(q_out, 16) || (s && !aligned(s, 16)) || !aligned(scale_out, 4) ||
        (mse_out && !aligned(mse_out, 8)) || (iters_out && !aligned(iters_out, 4)))
        return fail(SQ_ERR_ALIGN, "ssz_quant_weight: misaligned pointer (w, q_out, s need 16 bytes)");
    int sms;
    sq_status st = check_device(&sms);
    if (st != SQ_OK) return st;
    cudaStream_t cs = (cudaStream_t)stream;
    const bool bf = wt == SQ_BF16;
#define SSZ_LAUNCH(E)                                                                              \
    (bf ? launch_ssz<__nv_bfloat16, E>(w, N, K, s, bits, max_iters, q_out, scale_out, mse_out,     \
                                       iters_out, sms, cs)                                         \
        : launch_ssz<float, E>(w, N, K, s, bits, max_iters, q_out, scale_out, mse_out, iters_out, \
                               sms, cs))
    // elements per thread: at most 512 threads per channel row
    if (K <= 512) SSZ_LAUNCH(8);
    else if (K <= 2048) SSZ_LAUNCH(16);
    else if (K <= W8A8_SSZ_MID_MAX_K) SSZ_LAUNCH(W8A8_SSZ_MID_E);
    else if (K <= 16384) SSZ_LAUNCH(32);
    else SSZ_LAUNCH(64);
#undef SSZ_LAUNCH
    return launch_status("ssz_kernel");
}
