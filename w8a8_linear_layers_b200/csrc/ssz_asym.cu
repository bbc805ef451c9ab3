// ssz_asym.cu -- asymmetric per-output-channel int8 weight quantization with
// the SSZ search over scale and offset.
//
// Source: "SSZ：权重量化算法说明" (msModelSlim docs): 初始化阶段 (the MinMax
// observer's min/max give the initial scale and offset), 迭代优化阶段
// (asymmetric: scale and offset are optimised together by least squares;
// greedy keep), 收敛判断 and 算法参数 as in the symmetric search; 使用限制:
// asymmetric int4 is not supported, so this is int8 only.  The SmoothQuant
// fold W' = W diag(s) ("SmoothQuant大模型量化技术深度解析", section 1) is
// applied as the row is loaded.
//
// Reading (shared with the CPU oracle): the offset m lives in the weight
// domain, w ~ S u + m with u = clamp(rint(fl(w - m) / S), 0, 255), stored as
// the int8 code q = u - 128.  MinMax: m = min w, S = max((max w - min w) /
// 255, 1e-5).  A round fits w ~ a u + b to the kept codes in closed form,
//     den = K sum u^2 - (sum u)^2,  a = (K sum wu - sum w sum u) / den,
//     b = (sum w - a sum u) / K     (fp64; den == 0 keeps the pair),
// candidate S = max(fp32(a), 1e-5), m = fp32(b); error = mean over K of
// (w - (S u + m))^2 after re-quantising at the candidate; convergence and
// the greedy keep as in the symmetric search.
//
// Design: the symmetric kernel's (one CTA per channel, folded fp32 row and
// one code buffer in shared memory, codes 8 at a time on the packed fast
// path, moved and near-tie chunks visited after the pass, a rejected
// candidate ends the search and the chunks it touched are restored).  The
// error is evaluated exactly from exact sums,
//     K e = W2 - 2 S NUM - 2 m SW + S^2 DEN + 2 S m SU + K m^2
// (W2 = sum w^2, SW = sum w, NUM = sum w u in double-double; SU = sum u and
// DEN = sum u^2 exact integers), each product formed with TwoProduct and
// the terms added in double-double; NUM, SU and DEN change only where a code
// moves.
#include "common.cuh"
#include "dd.cuh"

namespace w8a8 {
namespace asym {

constexpr double kThreshold = 1e-10;
constexpr float kMinScale = 1e-5f;
constexpr float kUmax = 255.0f;
// clamp bounds of u: t in [M, M + 255]; int16 pairs in [0, 255]
constexpr float kLo = kRoundMagic, kHi = kRoundMagic + 255.0f;
constexpr uint32_t kLo2 = 0x00000000u, kHi2 = 0x00FF00FFu;

__device__ __forceinline__ int ubyte(uint2 p, int b) {
    const uint32_t w = b < 4 ? p.x : p.y;
    return (int)((w >> (8 * (b & 3))) & 0xffu);
}

// The exact code of one element (IEEE quotient), out of line: only taken for
// the rare elements near a rounding tie.
static __device__ __noinline__ int exact_ucode(float v, float S) {
    return (int)fminf(fmaxf(rintf(__fdiv_rn(v, S)), 0.0f), kUmax);
}

struct Sums {
    dd num;          // sum w u (init) or its change
    dd w2, sw;       // init only
    long long su;    // sum u or its change
    long long den;   // sum u^2 or its change
    bool moved;
    uint32_t touched;
};

// K e(S, m) from exact sums; below the evaluation error (a few 2^-100 W2)
// the error is zero.
__device__ __forceinline__ double error_k(dd W2, dd SW, dd NUM, long long SU, long long DEN, float S, float m,
                                          int K) {
    const double Sd = (double)S, md = (double)m;
    dd acc = W2;
    acc = dd_add(acc, dd_mul_d(NUM, -2.0 * Sd));
    acc = dd_add(acc, dd_mul_d(SW, -2.0 * md));
    acc = dd_add(acc, two_prod(Sd * Sd, (double)DEN));           // S^2 exact in fp64
    acc = dd_add(acc, two_prod(2.0 * Sd * md, (double)SU));      // 2 S m exact in fp64
    acc = dd_add(acc, two_prod(md * md, (double)K));             // m^2 exact in fp64
    const double v = acc.hi + acc.lo;
    return fabs(v) <= W2.hi * 0x1p-96 ? 0.0 : v;
}

// Least-squares candidate (S, m) from the kept sums, as the oracle forms it.
__device__ __forceinline__ void ls_candidate(dd NUM, dd SW, long long SU, long long DEN, int K, float keep_S,
                                             float keep_m, float &S, float &m) {
    const long long den_i = (long long)K * DEN - SU * SU;  // exact (< 2^63 for K <= 32768)
    if (den_i == 0) {
        S = keep_S;
        m = keep_m;
        return;
    }
    const double swu = NUM.hi + NUM.lo, sw = SW.hi + SW.lo, su = (double)SU;
    const double a = ((double)K * swu - sw * su) / (double)den_i;
    const double b = (sw - a * su) / (double)K;
    S = fmaxf((float)a, kMinScale);
    m = (float)b;
}

struct Consts {
    float r, m, S, tie_bound;
    bool narrow;
};

// Per-pair constants of a pass.  vmax bounds this thread's |w - m| (its
// max |w| plus |m|).  Called by whole warps.
__device__ __forceinline__ Consts pass_consts(float S, float m, float wabs) {
    Consts k;
    k.S = S;
    k.m = m;
    k.r = __fdiv_rn(1.0f, S);  // S >= 1e-5: finite
    const float vmax = (wabs + fabsf(m)) * 1.0000002f;
    k.tie_bound = 0.5f - fmaf(vmax * k.r, 4.76837158203125e-07f, 2.384185791015625e-07f);
    k.narrow = __all_sync(0xffffffffu, vmax * k.r < 16384.0f);
    return k;
}

// Fast codes u of the chunk at j: v = fl(w - m), then fast_codes8 on v.
template <bool NARROW>
__device__ __forceinline__ uint2 chunk_ucodes(const float *__restrict__ wrow, int j, const Consts &k,
                                              float &dmax) {
    const float4 a = *reinterpret_cast<const float4 *>(wrow + j);
    const float4 b = *reinterpret_cast<const float4 *>(wrow + j + 4);
    const float2 m2 = make_float2(k.m, k.m);
    const float2 v0 = f2_sub(make_float2(a.x, a.y), m2), v1 = f2_sub(make_float2(a.z, a.w), m2);
    const float2 v2 = f2_sub(make_float2(b.x, b.y), m2), v3 = f2_sub(make_float2(b.z, b.w), m2);
    return fast_codes8<NARROW>(make_float4(v0.x, v0.y, v1.x, v1.y), make_float4(v2.x, v2.y, v3.x, v3.y), k.r,
                               kLo, kHi, kLo2, kHi2, dmax);
}

// Main loop of a pass over this thread's chunks (as the symmetric search):
// init writes the codes and accumulates every sum; update only marks the
// chunks whose codes moved.  Both mark near-tie chunks.
template <bool INIT, bool NARROW>
__device__ __forceinline__ void pass_chunks(const float *__restrict__ wrow, int K, const Consts &k,
                                            uint8_t *__restrict__ u, Sums &out, uint32_t &moved, uint32_t &tie) {
    const int stride = blockDim.x * 8;
    int c = 0;
#pragma unroll 2
    for (int j = threadIdx.x * 8; j < K; j += stride, ++c) {
        float dmax = 0.0f;
        const uint2 nw = chunk_ucodes<NARROW>(wrow, j, k, dmax);
        if (dmax >= k.tie_bound) tie |= 1u << c;
        if (INIT) {
            *reinterpret_cast<uint2 *>(u + j) = nw;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int uu = ubyte(nw, i);
                const double wd = (double)wrow[j + i];
                dd_acc(out.w2, wd * wd);                // exact product
                dd_acc(out.sw, wd);
                dd_acc(out.num, wd * (double)uu);       // exact product
                out.su += uu;
                out.den += uu * uu;
            }
        } else {
            const uint2 od = *reinterpret_cast<const uint2 *>(u + j);
            if ((nw.x ^ od.x) | (nw.y ^ od.y)) moved |= 1u << c;
        }
    }
}

// Moved chunks: the change of NUM, SU and DEN, and the new codes written
// over the kept ones.
template <bool NARROW>
__device__ __forceinline__ void rewrite_moved(const float *__restrict__ wrow, uint32_t moved, const Consts &k,
                                              uint8_t *__restrict__ u, Sums &out) {
    const int stride = blockDim.x * 8;
    while (moved) {
        const int c = __ffs(moved) - 1;
        moved &= moved - 1u;
        const int j = threadIdx.x * 8 + c * stride;
        float dmax = 0.0f;
        const uint2 nw = chunk_ucodes<NARROW>(wrow, j, k, dmax);
        const uint2 od = *reinterpret_cast<const uint2 *>(u + j);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int un = ubyte(nw, i), uo = ubyte(od, i);
            if (un != uo) {
                out.su += un - uo;
                out.den += un * un - uo * uo;
                dd_acc(out.num, (double)wrow[j + i] * (double)(un - uo));  // exact product
            }
        }
        *reinterpret_cast<uint2 *>(u + j) = nw;
    }
}

// Near-tie chunks: the exact quotient decides their flagged elements, whose
// fast codes are already in u; with SUMS the sums follow.
template <bool SUMS>
__device__ __forceinline__ void fix_ties(const float *__restrict__ wrow, uint32_t tie, const Consts &k,
                                         uint8_t *__restrict__ u, Sums &out) {
    const int stride = blockDim.x * 8;
    while (tie) {
        const int c = __ffs(tie) - 1;
        tie &= tie - 1u;
        const int j = threadIdx.x * 8 + c * stride;
#pragma unroll 1
        for (int i = 0; i < 8; ++i) {
            const float w = wrow[j + i];
            const float v = __fsub_rn(w, k.m);
            const float t = fmaf(v, k.r, kRoundMagic);
            const float rq = t - kRoundMagic;
            const float d = fmaf(v, k.r, -rq);
            if (fabsf(d) + fmaf(fabsf(rq), 4.76837158203125e-07f, 2.384185791015625e-07f) >= 0.5f) {
                const int uf = (int)u[j + i];
                const int ue = exact_ucode(v, k.S);
                if (ue != uf) {
                    u[j + i] = (uint8_t)ue;
                    if (SUMS) {
                        out.su += ue - uf;
                        out.den += ue * ue - uf * uf;
                        dd_acc(out.num, (double)w * (double)(ue - uf));
                        out.moved = true;
                    }
                }
            }
        }
    }
}

template <bool INIT>
__device__ __forceinline__ Sums row_pass(const float *__restrict__ wrow, int K, float S, float m, float wabs,
                                         uint8_t *__restrict__ u) {
    const Consts k = pass_consts(S, m, wabs);
    Sums out = {{0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}, 0, 0, false, 0u};
    uint32_t moved = 0u, tie = 0u;
    if (k.narrow) pass_chunks<INIT, true>(wrow, K, k, u, out, moved, tie);
    else pass_chunks<INIT, false>(wrow, K, k, u, out, moved, tie);
    if (!INIT) {
        out.moved = moved != 0u;
        out.touched = moved | tie;
        if (k.narrow) rewrite_moved<true>(wrow, moved, k, u, out);
        else rewrite_moved<false>(wrow, moved, k, u, out);
    }
    fix_ties<true>(wrow, tie, k, u, out);
    return out;
}

// Exact codes at (S, m) over the chunks named in `touched`.
__device__ __forceinline__ void restore_chunks(const float *__restrict__ wrow, uint32_t touched, float S, float m,
                                               float wabs, uint8_t *__restrict__ u) {
    const Consts k = pass_consts(S, m, wabs);
    const int stride = blockDim.x * 8;
    uint32_t tie = 0u;
    for (uint32_t t = touched; t;) {
        const int c = __ffs(t) - 1;
        t &= t - 1u;
        const int j = threadIdx.x * 8 + c * stride;
        float dmax = 0.0f;
        const uint2 nw = k.narrow ? chunk_ucodes<true>(wrow, j, k, dmax) : chunk_ucodes<false>(wrow, j, k, dmax);
        if (dmax >= k.tie_bound) tie |= 1u << c;
        *reinterpret_cast<uint2 *>(u + j) = nw;
    }
    Sums unused;
    fix_ties<false>(wrow, tie, k, u, unused);
}

struct Part {
    dd num, w2, sw;
    long long su, den;
};

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <typename T, bool FOLD>
__global__ void __launch_bounds__(512)
ssz_asym_kernel(const T *__restrict__ wg, int64_t N, int K, const float *__restrict__ s, int max_iters,
                int8_t *__restrict__ q_out, float *__restrict__ scale_out, float *__restrict__ offset_out,
                double *__restrict__ mse_out, int32_t *__restrict__ iters_out) {
    extern __shared__ __align__(16) uint8_t smem[];
    float *wrow = reinterpret_cast<float *>(smem);         // K floats: the folded row
    uint8_t *u = reinterpret_cast<uint8_t *>(wrow + K);    // K codes u in [0, 255]: the kept codes
    __shared__ Part part[2][16];                           // per-warp partials, by round parity
    __shared__ float redlo[16], redhi[16];
    const int T_ = blockDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = T_ >> 5;
    const double kd = (double)K;
    const double thr_k = kThreshold * kd;

    for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
        // ---- stage the folded row; min, max and this thread's max |w|
        float lo = INFINITY, hi = -INFINITY, wabs = 0.0f;
#pragma unroll 4
        for (int j = threadIdx.x * 8; j < K; j += T_ * 8) {
            float v[8];
            Vec8<T>::load(wg + n * K + j, v);
            if (FOLD) {
                float f[8];
                load8_f32(s + j, f);
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = v[i] * f[i];
            }
            dbg_check8(v);  // the (smoothed) weights the search reads
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                lo = fminf(lo, v[i]);
                hi = fmaxf(hi, v[i]);
                wabs = fmaxf(wabs, fabsf(v[i]));
            }
            float4 *dst = reinterpret_cast<float4 *>(wrow + j);
            dst[0] = make_float4(v[0], v[1], v[2], v[3]);
            dst[1] = make_float4(v[4], v[5], v[6], v[7]);
        }
        lo = warp_min(lo);
        hi = warp_max(hi);
        if (lane == 0) {
            redlo[warp] = lo;
            redhi[warp] = hi;
        }
        __syncthreads();
        lo = redlo[0];
        hi = redhi[0];
        for (int i = 1; i < nwarps; ++i) {
            lo = fminf(lo, redlo[i]);
            hi = fmaxf(hi, redhi[i]);
        }

        // ---- MinMax init: m = min, S = (max - min) / 255 (floored)
        float S_best = fmaxf(__fdiv_rn(__fsub_rn(hi, lo), kUmax), kMinScale);
        float m_best = lo;
        int par = 0;
        {
            Sums p = row_pass<true>(wrow, K, S_best, m_best, wabs, u);
            p.num = warp_sum_dd(p.num);
            p.w2 = warp_sum_dd(p.w2);
            p.sw = warp_sum_dd(p.sw);
            p.su = warp_sum_ll(p.su);
            p.den = warp_sum_ll(p.den);
            if (lane == 0) part[par][warp] = {p.num, p.w2, p.sw, p.su, p.den};
        }
        __syncthreads();
        dd W2 = part[par][0].w2, SW = part[par][0].sw, NUM = part[par][0].num;
        long long SU = part[par][0].su, DEN = part[par][0].den;
        for (int i = 1; i < nwarps; ++i) {
            W2 = dd_add_cascade(W2, part[par][i].w2);
            SW = dd_add_cascade(SW, part[par][i].sw);
            NUM = dd_add_cascade(NUM, part[par][i].num);
            SU += part[par][i].su;
            DEN += part[par][i].den;
        }
        double e_best = error_k(W2, SW, NUM, SU, DEN, S_best, m_best, K);  // K x error
        float S_c, m_c;
        ls_candidate(NUM, SW, SU, DEN, K, S_best, m_best, S_c, m_c);
        int it = 0;
        bool done = max_iters == 0;
        uint32_t touched = 0u;
        bool rejected = false;

        // ---- least-squares rounds (a candidate that is not kept ends the search)
        while (!done) {
            par ^= 1;
            Sums p = row_pass<false>(wrow, K, S_c, m_c, wabs, u);
            touched = p.touched;
            if (__any_sync(0xffffffffu, p.moved)) {
                p.num = warp_sum_dd(p.num);
                p.su = warp_sum_ll(p.su);
                p.den = warp_sum_ll(p.den);
            } else {
                p.num = {0.0, 0.0};
                p.su = 0;
                p.den = 0;
            }
            if (lane == 0) part[par][warp] = {p.num, {0.0, 0.0}, {0.0, 0.0}, p.su, p.den};
            __syncthreads();
            ++it;
            dd num_c = NUM;
            long long su_c = SU, den_c = DEN;
            for (int i = 0; i < nwarps; ++i) {
                num_c = dd_add_cascade(num_c, part[par][i].num);
                su_c += part[par][i].su;
                den_c += part[par][i].den;
            }
            const double e_c = error_k(W2, SW, num_c, su_c, den_c, S_c, m_c, K);
            float S_n, m_n;
            ls_candidate(num_c, SW, su_c, den_c, K, S_c, m_c, S_n, m_n);  // used only if kept
            const double delta = e_best - e_c;
            done = (e_best == 0.0) || (delta < kThreshold * e_best) || (fabs(delta) < thr_k) || it == max_iters;
            if (e_c < e_best) {
                S_best = S_c;
                m_best = m_c;
                e_best = e_c;
                NUM = num_c;
                SU = su_c;
                DEN = den_c;
                S_c = S_n;
                m_c = m_n;
            } else {
                rejected = true;
                done = true;  // implied by the tests above (e_best >= 0); stated for the restore below
            }
        }
        if (rejected) restore_chunks(wrow, touched, S_best, m_best, wabs, u);

        // ---- kept codes out as q = u - 128 (each thread its own chunks)
        for (int j = threadIdx.x * 8; j < K; j += T_ * 8) {
            uint2 c = *reinterpret_cast<const uint2 *>(u + j);
            c.x ^= 0x80808080u;
            c.y ^= 0x80808080u;
            *reinterpret_cast<uint2 *>(q_out + n * K + j) = c;
        }
        if (threadIdx.x == 0) {
            scale_out[n] = S_best;
            offset_out[n] = m_best;
            if (mse_out) mse_out[n] = e_best / kd;
            if (iters_out) iters_out[n] = it;
        }
        __syncthreads();  // shared row and codes are reused by the next channel
    }
}

template <typename T>
static sq_status launch(const void *w, int64_t N, int64_t K, const float *s, int max_iters, int8_t *q,
                        float *scale, float *offset, double *mse, int32_t *iters, int sms, cudaStream_t st) {
    // warps per channel: one per 2048 elements, at most 32 chunks per thread
    int64_t wps = std::max<int64_t>(ceil_div(K, 2048), ceil_div(K, 32 * 32 * 8));
    const int threads = 32 * (int)std::min<int64_t>(16, std::max<int64_t>(1, wps));
    const size_t smem = 5 * (size_t)K;  // fp32 row + codes
    auto kern = s ? ssz_asym_kernel<T, true> : ssz_asym_kernel<T, false>;
    if (smem > 32 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    }
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
    const int64_t grid = std::min<int64_t>(N, (int64_t)sms * std::max(per_sm, 1) * 8);
    kern<<<(unsigned)grid, threads, smem, st>>>((const T *)w, N, (int)K, s, max_iters, q, scale, offset, mse,
                                               iters);
    return launch_status("ssz_asym_kernel");
}

}  // namespace asym
W8A8_DEBUG_READER(ssz_asym)

}  // namespace w8a8

using namespace w8a8;

extern "C" sq_status ssz_quant_weight_asym(const void *w, sq_dtype wt, int64_t N, int64_t K, const float *s,
                                           int max_iters, int8_t *q_out, float *scale_out, float *offset_out,
                                           double *mse_out, int32_t *iters_out, void *stream) {
    if (N > 0 && (!w || !q_out || !scale_out || !offset_out))
        return fail(SQ_ERR_NULL, "ssz_quant_weight_asym: NULL pointer");
    if (wt != SQ_F32 && wt != SQ_BF16) return fail(SQ_ERR_DTYPE, "ssz_quant_weight_asym: dtype %d", (int)wt);
    if (N < 0 || K <= 0 || K % 16 != 0 || K > 32768)
        return fail(SQ_ERR_SHAPE, "ssz_quant_weight_asym: N=%lld K=%lld (K must be a multiple of 16 in [16, 32768])",
                    (long long)N, (long long)K);
    if (max_iters < 0 || max_iters > 255)
        return fail(SQ_ERR_ARG, "ssz_quant_weight_asym: max_iters=%d outside [0, 255]", max_iters);
    if (N == 0) return SQ_OK;
    if (!aligned(w, 16) || !aligned(q_out, 16) || (s && !aligned(s, 16)) || !aligned(scale_out, 4) ||
        !aligned(offset_out, 4) || (mse_out && !aligned(mse_out, 8)) || (iters_out && !aligned(iters_out, 4)))
        return fail(SQ_ERR_ALIGN, "ssz_quant_weight_asym: misaligned pointer");
    int sms;
    sq_status st = check_device(&sms);
    if (st != SQ_OK) return st;
    cudaStream_t cs = (cudaStream_t)stream;
    if (wt == SQ_BF16)
        return asym::launch<__nv_bfloat16>(w, N, K, s, max_iters, q_out, scale_out, offset_out, mse_out, iters_out,
                                           sms, cs);
    return asym::launch<float>(w, N, K, s, max_iters, q_out, scale_out, offset_out, mse_out, iters_out, sms, cs);
}
