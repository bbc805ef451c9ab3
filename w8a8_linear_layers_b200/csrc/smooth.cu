// smooth.cu -- steps 1 and 2 of the SmoothQuant W8A8 path.
//
//  sq_calib_absmax : per-input-channel activation absmax, max|X_j| of the
//                    SmoothQuant smoothing factor ("SmoothQuant大模型量化技术
//                    深度解析", section 1), gathered over calibration batches
//                    ("训练后量化（PTQ）", PTQ 的基本流程).
//  sq_smooth_fold  : max|W_j| over the input channel j of W, then
//                    s_j = max|X_j|^a / max|W_j|^(1-a) and 1/s_j (same section),
//                    and optionally W * diag(s) materialized in fp32.
//
// Both reductions are column maxima of a row-major matrix: HBM-bound, one
// read of the matrix.  Each thread streams 16-byte vectors of 8 (bf16) or 4
// (fp32) consecutive columns down a slice of rows, keeping its running maxima
// in registers; a CTA folds its 8 warps in shared memory and merges into the
// [K] result with an integer atomicMax on the fp32 bit pattern (valid for the
// non-negative values |x|; max is exact and order-free, so the result is
// bit-identical to a sequential scan).
#include "common.cuh"

#include <math.h>

namespace w8a8 {

constexpr int kColThreads = 256;
constexpr int kColWarps = kColThreads / 32;
constexpr int kColDepth = 6;  // row loads in flight per thread

template <typename T> struct ColVec;
template <> struct ColVec<__nv_bfloat16> { static constexpr int N = 8; };
template <> struct ColVec<float> { static constexpr int N = 4; };

// A 16-byte vector of VEC consecutive columns, raw, and its |.| folded into
// the running maxima m.
template <typename T> struct ColRaw;
template <> struct ColRaw<__nv_bfloat16> { using type = uint4; };
template <> struct ColRaw<float> { using type = float4; };

template <typename T>
__device__ __forceinline__ typename ColRaw<T>::type load_raw(const T *p) {
    return __ldg(reinterpret_cast<const typename ColRaw<T>::type *>(p));
}

__device__ __forceinline__ void fold_abs(float (&m)[8], uint4 u) {
    dbg_check_bf16x8(u);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        m[2 * i] = fmaxf(m[2 * i], __uint_as_float((w[i] << 16) & 0x7fff0000u));
        m[2 * i + 1] = fmaxf(m[2 * i + 1], __uint_as_float(w[i] & 0x7fff0000u));
    }
}

__device__ __forceinline__ void fold_abs(float (&m)[4], float4 a) {
    dbg_check4(a);
    m[0] = fmaxf(m[0], fabsf(a.x));
    m[1] = fmaxf(m[1], fabsf(a.y));
    m[2] = fmaxf(m[2], fabsf(a.z));
    m[3] = fmaxf(m[3], fabsf(a.w));
}

// grid.x: column strips of 32 * VEC columns; grid.y: row slices.
// out_bits: [K] fp32 maxima viewed as unsigned ints (non-negative floats
// order like their bit patterns).
template <typename T>
__global__ void __launch_bounds__(kColThreads, 4)
col_absmax_kernel(const T *__restrict__ a, int64_t R, int64_t K, int64_t rows_per_slice,
                  unsigned int *__restrict__ out_bits) {
    constexpr int VEC = ColVec<T>::N;
    constexpr int STRIP = 32 * VEC;
    __shared__ float red[kColWarps][STRIP];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t col = (int64_t)blockIdx.x * STRIP + lane * VEC;
    const int64_t r0 = (int64_t)blockIdx.y * rows_per_slice;
    const int64_t r1 = min(R, r0 + rows_per_slice);

    float m[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) m[i] = 0.0f;

    if (col < K) {
        const T *p = a + col;
        // up to kColDepth independent 16-byte loads in flight per thread: a
        // slice is a few dozen rows deep, so one or two round trips cover it
        for (int64_t r = r0 + warp; r < r1; r += kColDepth * kColWarps) {
            typename ColRaw<T>::type v[kColDepth];
#pragma unroll
            for (int u = 0; u < kColDepth; ++u) {
                const int64_t rr = r + u * kColWarps;
                if (rr < r1 && dbg_index_ok(rr < R && col + VEC <= K)) v[u] = load_raw<T>(p + rr * K);
            }
#pragma unroll
            for (int u = 0; u < kColDepth; ++u)
                if (r + u * kColWarps < r1 && dbg_index_again(r + u * kColWarps < R && col + VEC <= K))
                    fold_abs(m, v[u]);
        }
    }
#pragma unroll
    for (int i = 0; i < VEC; ++i) red[warp][lane * VEC + i] = m[i];
    __syncthreads();
    for (int c = threadIdx.x; c < STRIP; c += kColThreads) {
        int64_t j = (int64_t)blockIdx.x * STRIP + c;
        if (j >= K) continue;
        float v = red[0][c];
#pragma unroll
        for (int w = 1; w < kColWarps; ++w) v = fmaxf(v, red[w][c]);
        atomicMax(out_bits + j, __float_as_uint(v));
    }
}

static sq_status launch_col_absmax(const void *a, sq_dtype t, int64_t R, int64_t K,
                                   float *out, bool accumulate, int sms, cudaStream_t st) {
    if (!accumulate) {
        cudaError_t e = cudaMemsetAsync(out, 0, (size_t)K * sizeof(float), st);
        if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "memset: %s", cudaGetErrorString(e));
    }
    if (R == 0) return SQ_OK;
    const int vec = (t == SQ_BF16) ? 8 : 4;
    const int64_t strips = ceil_div(K, 32 * vec);
    // about four CTAs per SM, each slice at least 32 rows deep
    int64_t slices = ceil_div(4LL * sms, strips);
    slices = std::max<int64_t>(1, std::min<int64_t>(slices, ceil_div(R, 32)));
    slices = std::min<int64_t>(slices, 65535);
    const int64_t rows = ceil_div(R, slices);
    slices = ceil_div(R, rows);
    dim3 grid((unsigned)strips, (unsigned)slices);
    if (t == SQ_BF16)
        col_absmax_kernel<__nv_bfloat16><<<grid, kColThreads, 0, st>>>(
            (const __nv_bfloat16 *)a, R, K, rows, (unsigned int *)out);
    else
        col_absmax_kernel<float><<<grid, kColThreads, 0, st>>>(
            (const float *)a, R, K, rows, (unsigned int *)out);
    return launch_status("col_absmax_kernel");
}

// s_j = fp32(ax^alpha / aw^(1-alpha)) in fp64, 1 for an empty channel;
// inv_s_j = 1/s_j with an IEEE fp32 division.
__global__ void smooth_factor_kernel(const float *__restrict__ ax, const float *__restrict__ aw,
                                     int64_t K, float alpha, float *__restrict__ s,
                                     float *__restrict__ inv_s) {
    int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= K) return;
    float a = ax[j], b = aw[j];
    float sj;
    if (a == 0.0f || b == 0.0f) {
        sj = 1.0f;
    } else {
        double al = (double)alpha;
        sj = (float)(pow((double)a, al) / pow((double)b, 1.0 - al));
    }
    s[j] = sj;
    inv_s[j] = __fdiv_rn(1.0f, sj);
}

// w_folded[n, j] = w[n, j] * s[j] (one fp32 multiply), 8 columns per thread.
template <typename T>
__global__ void fold_kernel(const T *__restrict__ w, int64_t N, int64_t K,
                            const float *__restrict__ s, float *__restrict__ out) {
    const int64_t groups_per_row = K / 8;
    const int64_t total = N * groups_per_row;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total;
         g += (int64_t)gridDim.x * blockDim.x) {
        int64_t n = g / groups_per_row, j = (g - n * groups_per_row) * 8;
        float v[8], f[8];
        Vec8<T>::load(w + n * K + j, v);
        load8_f32(s + j, f);
        float4 *o = reinterpret_cast<float4 *>(out + n * K + j);
        o[0] = make_float4(v[0] * f[0], v[1] * f[1], v[2] * f[2], v[3] * f[3]);
        o[1] = make_float4(v[4] * f[4], v[5] * f[5], v[6] * f[6], v[7] * f[7]);
    }
}

W8A8_DEBUG_READER(smooth)

}  // namespace w8a8

using namespace w8a8;

extern "C" sq_status sq_calib_absmax(const void *x, sq_dtype xt, int64_t M, int64_t K,
                                     float *absmax, int accumulate, void *stream) {
    if (!absmax || (M > 0 && !x)) return fail(SQ_ERR_NULL, "sq_calib_absmax: NULL pointer");
    if (xt != SQ_F32 && xt != SQ_BF16) return fail(SQ_ERR_DTYPE, "sq_calib_absmax: dtype %d", (int)xt);
    if (M < 0 || K <= 0 || K % 16 != 0)
        return fail(SQ_ERR_SHAPE, "sq_calib_absmax: M=%lld K=%lld (K must be a positive multiple of 16)",
                    (long long)M, (long long)K);
    if ((x && !aligned(x, 16)) || !aligned(absmax, 4))
        return fail(SQ_ERR_ALIGN, "sq_calib_absmax: x must be 16-byte aligned");
    int sms;
    sq_status st = check_device(&sms);
    if (st != SQ_OK) return st;
    return launch_col_absmax(x, xt, M, K, absmax, accumulate != 0, sms, (cudaStream_t)stream);
}

extern "C" sq_status sq_smooth_fold(const float *x_absmax, const void *w, sq_dtype wt, int64_t N,
                                    int64_t K, float alpha, float *w_absmax_out, float *s_out,
                                    float *inv_s_out, float *w_folded_out, void *stream) {
    if (!x_absmax || !w_absmax_out || !s_out || !inv_s_out || (N > 0 && !w))
        return fail(SQ_ERR_NULL, "sq_smooth_fold: NULL pointer");
    if (wt != SQ_F32 && wt != SQ_BF16) return fail(SQ_ERR_DTYPE, "sq_smooth_fold: dtype %d", (int)wt);
    if (N < 0 || K <= 0 || K % 16 != 0)
        return fail(SQ_ERR_SHAPE, "sq_smooth_fold: N=%lld K=%lld (K must be a positive multiple of 16)",
                    (long long)N, (long long)K);
    if (!(alpha >= 0.0f && alpha <= 1.0f))
        return fail(SQ_ERR_ARG, "sq_smooth_fold: alpha=%g outside [0,1]", (double)alpha);
    if ((w && !aligned(w, 16)) || (w_folded_out && !aligned(w_folded_out, 16)) ||
        !aligned(x_absmax, 4) || !aligned(w_absmax_out, 4) || !aligned(s_out, 4) || !aligned(inv_s_out, 4))
        return fail(SQ_ERR_ALIGN, "sq_smooth_fold: misaligned pointer");
    // the fold reads s eight columns at a time with 16-byte loads
    if (w_folded_out && !aligned(s_out, 16))
        return fail(SQ_ERR_ALIGN, "sq_smooth_fold: s_out must be 16-byte aligned when w_folded_out is given");
    int sms;
    sq_status st = check_device(&sms);
    if (st != SQ_OK) return st;
    cudaStream_t cs = (cudaStream_t)stream;
    st = launch_col_absmax(w, wt, N, K, w_absmax_out, false, sms, cs);
    if (st != SQ_OK) return st;
    smooth_factor_kernel<<<(unsigned)ceil_div(K, 256), 256, 0, cs>>>(x_absmax, w_absmax_out, K, alpha,
                                                                     s_out, inv_s_out);
    st = launch_status("smooth_factor_kernel");
    if (st != SQ_OK || !w_folded_out || N == 0) return st;
    const int64_t groups = N * (K / 8);
    const unsigned blocks = (unsigned)std::min<int64_t>(ceil_div(groups, 256), 8LL * sms);
    if (wt == SQ_BF16)
        fold_kernel<__nv_bfloat16><<<blocks, 256, 0, cs>>>((const __nv_bfloat16 *)w, N, K, s_out, w_folded_out);
    else
        fold_kernel<float><<<blocks, 256, 0, cs>>>((const float *)w, N, K, s_out, w_folded_out);
    return launch_status("fold_kernel");
}

extern "C" sq_status sq_smooth_factor(const float *x_absmax, const float *w_absmax, int64_t K, float alpha,
                                      float *s_out, float *inv_s_out, void *stream) {
    if (!x_absmax || !w_absmax || !s_out || !inv_s_out) return fail(SQ_ERR_NULL, "sq_smooth_factor: NULL pointer");
    if (K <= 0 || K % 16 != 0)
        return fail(SQ_ERR_SHAPE, "sq_smooth_factor: K=%lld (a positive multiple of 16)", (long long)K);
    if (!(alpha >= 0.0f && alpha <= 1.0f))
        return fail(SQ_ERR_ARG, "sq_smooth_factor: alpha=%g outside [0,1]", (double)alpha);
    if (!aligned(x_absmax, 4) || !aligned(w_absmax, 4) || !aligned(s_out, 4) || !aligned(inv_s_out, 4))
        return fail(SQ_ERR_ALIGN, "sq_smooth_factor: misaligned pointer");
    int sms;
    sq_status st = check_device(&sms);
    if (st != SQ_OK) return st;
    smooth_factor_kernel<<<(unsigned)ceil_div(K, 256), 256, 0, (cudaStream_t)stream>>>(x_absmax, w_absmax, K, alpha,
                                                                                      s_out, inv_s_out);
    return launch_status("smooth_factor_kernel");
}
