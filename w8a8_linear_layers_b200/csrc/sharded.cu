// sharded.cu -- the two kernels the row-parallel (K-sharded) linear needs
// beyond the five steps.
//
// With K split across ranks, every rank computes its slice's per-token
// scales (quant_act_per_token), the ranks take the MAX of those scales (the
// map a -> fl(a / 127) is monotonic, so the MAX is the unsharded scale),
// quantize their slices at that scale (quant_act_given_scale), multiply
// (w8a8_gemm_dequant with acc_out), SUM the int32 accumulators (exact), and
// dequantize the sum (sq_dequant).  Sources: the per-token quantization and
// dequant of the CUDA INT8 notes (aicoding.csdn.net), sections 2.1 and 4.2;
// the SmoothQuant fold ("SmoothQuant大模型量化技术深度解析", section 1).
#include "common.cuh"

namespace w8a8 {
namespace shard {

// One thread per 8 consecutive elements of a row (grid-stride over the
// matrix); the row's scale is read from sx.
template <typename T>
__global__ void quant_given_kernel(const T *__restrict__ x, int64_t M, int64_t K, const float *__restrict__ inv_s,
                                   const float *__restrict__ sx, int8_t *__restrict__ q) {
    const int64_t per_row = K / 8;
    const int64_t total = M * per_row;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total;
         g += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = g / per_row, j = (g - t * per_row) * 8;
        float v[8];
        Vec8<T>::load(x + t * K + j, v);
        if (inv_s) {
            float f[8];
            load8_f32(inv_s + j, f);
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = v[i] * f[i];
        }
        const float s = sx[t];
        int code[8];
        if (s == 0.0f) {
#pragma unroll
            for (int i = 0; i < 8; ++i) code[i] = 0;
        } else {
            const float r = __fdiv_rn(1.0f, s);
            const bool exact_only = !(fabsf(r) <= 3.402823466e38f);  // 1/s overflowed
#pragma unroll
            for (int i = 0; i < 8; ++i) code[i] = (int)sym_code(v[i], s, r, 127.0f, exact_only);
        }
        *reinterpret_cast<uint2 *>(q + t * K + j) = pack8_codes(code);
    }
}

// y = ((float)acc * sx[row]) * sw[col], 4 columns per thread.
template <typename OutT>
__global__ void dequant_kernel(const int32_t *__restrict__ acc, const float *__restrict__ sx,
                               const float *__restrict__ sw, int64_t M, int64_t N, OutT *__restrict__ y) {
    const int64_t per_row = N / 4;
    const int64_t total = M * per_row;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total;
         g += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = g / per_row, n = (g - t * per_row) * 4;
        const int4 a = __ldg(reinterpret_cast<const int4 *>(acc + t * N + n));
        const float4 w = __ldg(reinterpret_cast<const float4 *>(sw + n));
        const float s = sx[t];
        const float v0 = (__int2float_rn(a.x) * s) * w.x, v1 = (__int2float_rn(a.y) * s) * w.y;
        const float v2 = (__int2float_rn(a.z) * s) * w.z, v3 = (__int2float_rn(a.w) * s) * w.w;
        if (sizeof(OutT) == 2) {
            __nv_bfloat162 lo = __floats2bfloat162_rn(v0, v1), hi = __floats2bfloat162_rn(v2, v3);
            *reinterpret_cast<uint2 *>(y + t * N + n) =
                make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
        } else {
            *reinterpret_cast<float4 *>(y + t * N + n) = make_float4(v0, v1, v2, v3);
        }
    }
}

}  // namespace shard
}  // namespace w8a8

using namespace w8a8;

extern "C" sq_status quant_act_given_scale(const void *x, sq_dtype xt, int64_t M, int64_t K, const float *inv_s,
                                           const float *sx, int8_t *q_out, void *stream) {
    if (M > 0 && (!x || !sx || !q_out)) return fail(SQ_ERR_NULL, "quant_act_given_scale: NULL pointer");
    if (xt != SQ_F32 && xt != SQ_BF16) return fail(SQ_ERR_DTYPE, "quant_act_given_scale: dtype %d", (int)xt);
    if (M < 0 || K <= 0 || K % 16 != 0)
        return fail(SQ_ERR_SHAPE, "quant_act_given_scale: M=%lld K=%lld (K a positive multiple of 16)",
                    (long long)M, (long long)K);
    if (M == 0) return SQ_OK;
    if (!aligned(x, 16) || !aligned(q_out, 16) || !aligned(sx, 4) || (inv_s && !aligned(inv_s, 16)))
        return fail(SQ_ERR_ALIGN, "quant_act_given_scale: misaligned pointer (x, q_out, inv_s need 16 bytes)");
    int sms;
    sq_status st = check_device(&sms);
    if (st != SQ_OK) return st;
    const int64_t units = M * (K / 8);
    const unsigned blocks = (unsigned)std::min<int64_t>(ceil_div(units, 256), 8LL * sms);
    if (xt == SQ_BF16)
        shard::quant_given_kernel<__nv_bfloat16><<<blocks, 256, 0, (cudaStream_t)stream>>>(
            (const __nv_bfloat16 *)x, M, K, inv_s, sx, q_out);
    else
        shard::quant_given_kernel<float><<<blocks, 256, 0, (cudaStream_t)stream>>>((const float *)x, M, K, inv_s,
                                                                                  sx, q_out);
    return launch_status("quant_given_kernel");
}

extern "C" sq_status sq_dequant(const int32_t *acc, const float *sx, const float *sw, int64_t M, int64_t N, void *y,
                                sq_dtype yt, void *stream) {
    if (M > 0 && N > 0 && (!acc || !sx || !sw || !y)) return fail(SQ_ERR_NULL, "sq_dequant: NULL pointer");
    if (yt != SQ_F32 && yt != SQ_BF16) return fail(SQ_ERR_DTYPE, "sq_dequant: output dtype %d", (int)yt);
    if (M < 0 || N < 0 || N % 4 != 0)
        return fail(SQ_ERR_SHAPE, "sq_dequant: M=%lld N=%lld (N a multiple of 4)", (long long)M, (long long)N);
    if (M == 0 || N == 0) return SQ_OK;
    if (!aligned(acc, 16) || !aligned(sw, 16) || !aligned(sx, 4) || !aligned(y, yt == SQ_BF16 ? 8 : 16))
        return fail(SQ_ERR_ALIGN, "sq_dequant: misaligned pointer (acc, sw 16 bytes; y 8 or 16)");
    int sms;
    sq_status st = check_device(&sms);
    if (st != SQ_OK) return st;
    const int64_t units = M * (N / 4);
    const unsigned blocks = (unsigned)std::min<int64_t>(ceil_div(units, 256), 8LL * sms);
    if (yt == SQ_BF16)
        shard::dequant_kernel<__nv_bfloat16><<<blocks, 256, 0, (cudaStream_t)stream>>>(acc, sx, sw, M, N,
                                                                                      (__nv_bfloat16 *)y);
    else
        shard::dequant_kernel<float><<<blocks, 256, 0, (cudaStream_t)stream>>>(acc, sx, sw, M, N, (float *)y);
    return launch_status("dequant_kernel");
}
