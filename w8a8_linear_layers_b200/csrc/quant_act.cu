// quant_act.cu -- step 4: per-token symmetric int8 activation quantization.
//
// Source: CUDA INT8 quantization notes (aicoding.csdn.net), section 2.1
// ("量化基础理论"): Q = round(R/S) + Z with range calibration, parameter
// computation and saturation; Z = 0 here (symmetric), one scale per token,
// round half to even and saturation to [-127, 127].  The SmoothQuant fold
// ("SmoothQuant大模型量化技术深度解析", section 1: activations divided by s)
// is applied on the fly as x * inv_s.
//
// Design: one CTA per token row (grid-stride), the row held in registers
// between its two uses (absmax, then codes), so X is read from HBM once and
// the codes written once: 2 (bf16) + 1 bytes per element.  Each thread owns
// E/8 chunks of 8 consecutive columns; chunk c of thread t starts at column
// (c * T + t) * 8, so a warp's loads are 512 contiguous bytes (bf16).
#include "common.cuh"

namespace w8a8 {

template <typename T, int E>
__global__ void __launch_bounds__(512)
quant_act_kernel(const T *__restrict__ x, int64_t M, int64_t K, const float *__restrict__ inv_s,
                 int8_t *__restrict__ q, float *__restrict__ scale) {
    constexpr int C = E / 8;  // chunks per thread
    // inv_s is kept in registers across rows unless that would spill (E = 64)
    constexpr bool kCacheInvS = C <= 4;
    __shared__ float red[2][32];
    const int T_ = blockDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = T_ >> 5;

    float f[kCacheInvS ? C : 1][8];  // inv_s for this thread's columns (constant across rows)
    bool live[C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
        int64_t j = ((int64_t)c * T_ + threadIdx.x) * 8;
        live[c] = j < K;
        if (kCacheInvS) {
            if (live[c] && inv_s) {
                load8_f32(inv_s + j, f[kCacheInvS ? c : 0]);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) f[kCacheInvS ? c : 0][i] = 1.0f;
            }
        }
    }

    int parity = 0;
    for (int64_t row = blockIdx.x; row < M; row += gridDim.x, parity ^= 1) {
        const T *xr = x + row * K;
        float v[C][8];
        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            if (live[c]) {
                Vec8<T>::load(xr + ((int64_t)c * T_ + threadIdx.x) * 8, v[c]);
                if (inv_s) {
                    if (!kCacheInvS) load8_f32(inv_s + ((int64_t)c * T_ + threadIdx.x) * 8, f[0]);
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[c][i] = v[c][i] * f[kCacheInvS ? c : 0][i];
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[c][i] = 0.0f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[c][i]));
        }
        amax = warp_max(amax);
        if (lane == 0) red[parity][warp] = amax;
        __syncthreads();  // red[parity] complete; red[parity^1] free for the next row
        amax = red[parity][0];
        for (int w = 1; w < nwarps; ++w) amax = fmaxf(amax, red[parity][w]);

        const float s = __fdiv_rn(amax, 127.0f);
        if (threadIdx.x == 0) scale[row] = s;
        const float r = __fdiv_rn(1.0f, s);
        const bool exact_only = !(fabsf(r) <= 3.402823466e38f);  // 1/s overflowed (or s == 0)
        int8_t *qr = q + row * K;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            if (!live[c]) continue;
            int code[8];
            if (s == 0.0f) {
#pragma unroll
                for (int i = 0; i < 8; ++i) code[i] = 0;
            } else if (exact_only) {
#pragma unroll
                for (int i = 0; i < 8; ++i) code[i] = (int)sym_code(v[c][i], s, r, 127.0f, true);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) code[i] = sym_code_i(v[c][i], s, r, 127.0f);
            }
            *reinterpret_cast<uint2 *>(qr + ((int64_t)c * T_ + threadIdx.x) * 8) = pack8_codes(code);
        }
    }
}

template <typename T, int E>
static void launch_quant_act(const void *x, int64_t M, int64_t K, const float *inv_s, int8_t *q,
                             float *scale, int sms, cudaStream_t st) {
    int threads = (int)ceil_div(ceil_div(K, E), 32) * 32;
    // enough CTAs to fill the machine; each strides over rows
    int per_sm = std::max(1, 2048 / threads);
    int64_t grid = std::min<int64_t>(M, (int64_t)sms * per_sm);
    quant_act_kernel<T, E><<<(unsigned)grid, threads, 0, st>>>((const T *)x, M, K, inv_s, q, scale);
}

}  // namespace w8a8

using namespace w8a8;

extern "C" sq_status quant_act_per_token(const void *x, sq_dtype xt, int64_t M, int64_t K,
                                         const float *inv_s, int8_t *q_out, float *scale_out,
                                         void *stream) {
    if (M > 0 && (!x || !q_out || !scale_out)) return fail(SQ_ERR_NULL, "quant_act_per_token: NULL pointer");
    if (xt != SQ_F32 && xt != SQ_BF16) return fail(SQ_ERR_DTYPE, "quant_act_per_token: dtype %d", (int)xt);
    if (M < 0 || K <= 0 || K % 16 != 0 || K > 32768)
        return fail(SQ_ERR_SHAPE, "quant_act_per_token: M=%lld K=%lld (K must be a multiple of 16 in [16, 32768])",
                    (long long)M, (long long)K);
    if (M == 0) return SQ_OK;
    if (!aligned(x, 16) || !aligned(q_out, 16) || !aligned(scale_out, 4) || (inv_s && !aligned(inv_s, 16)))
        return fail(SQ_ERR_ALIGN, "quant_act_per_token: misaligned pointer (x, q_out, inv_s need 16 bytes)");
    int sms;
    sq_status st = check_device(&sms);
    if (st != SQ_OK) return st;
    cudaStream_t cs = (cudaStream_t)stream;
    // elements per thread: at most 512 threads per row
    const bool bf = xt == SQ_BF16;
    if (K <= 2048) {
        if (bf) launch_quant_act<__nv_bfloat16, 8>(x, M, K, inv_s, q_out, scale_out, sms, cs);
        else launch_quant_act<float, 8>(x, M, K, inv_s, q_out, scale_out, sms, cs);
    } else if (K <= 8192) {
        if (bf) launch_quant_act<__nv_bfloat16, 16>(x, M, K, inv_s, q_out, scale_out, sms, cs);
        else launch_quant_act<float, 16>(x, M, K, inv_s, q_out, scale_out, sms, cs);
    } else if (K <= 16384) {
        if (bf) launch_quant_act<__nv_bfloat16, 32>(x, M, K, inv_s, q_out, scale_out, sms, cs);
        else launch_quant_act<float, 32>(x, M, K, inv_s, q_out, scale_out, sms, cs);
    } else {
        if (bf) launch_quant_act<__nv_bfloat16, 64>(x, M, K, inv_s, q_out, scale_out, sms, cs);
        else launch_quant_act<float, 64>(x, M, K, inv_s, q_out, scale_out, sms, cs);
    }
    return launch_status("quant_act_kernel");
}
