// quant_act.cu -- step 4: per-token symmetric int8 activation quantization,
// and its variants: static per-tensor scales (quant_act_static with
// sq_static_range_update), row sums of the codes for asymmetric weights, and
// the LayerNorm fused with the smoothing and the quantization
// (sq_layernorm_quant).
//
// Source: CUDA INT8 quantization notes (aicoding.csdn.net), section 2.1
// ("量化基础理论"): Q = round(R/S) + Z with range calibration, parameter
// computation and saturation; Z = 0 here (symmetric), one scale per token,
// round half to even and saturation to [-127, 127].  The SmoothQuant fold
// ("SmoothQuant大模型量化技术深度解析", section 1: activations divided by s)
// is applied on the fly as x * inv_s.
//
// Design: one small CTA per token row (grid-stride), the row held in
// registers between its two uses (absmax, then codes), so X is read from HBM
// once and the codes written once: 2 (bf16) + 1 bytes per element.  Each
// thread owns E/8 chunks of 8 consecutive columns; chunk c of thread t starts
// at column (c * T + t) * 8, so a warp's loads are 512 contiguous bytes
// (bf16).  Codes come 8 at a time from the packed fast path (fast_codes8);
// only chunks with an element near a rounding tie take the exact quotient.
#include "common.cuh"

namespace w8a8 {

// 8 consecutive elements as loaded (16 bytes of bf16 or 32 bytes of fp32),
// widened to fp32 only where used, so a CTA can keep several rows in flight.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    uint4 u;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) { u = __ldg(reinterpret_cast<const uint4 *>(p)); }
    __device__ __forceinline__ void zero() { u = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void widen(float (&v)[8]) const {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};
template <> struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float *p) {
        a = __ldg(reinterpret_cast<const float4 *>(p));
        b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void widen(float (&v)[8]) const {
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

// Clamp bounds of the int8 codes: t in [M - 127, M + 127]; int16 pairs in
// [-127, 127].
constexpr float kLo = kRoundMagic - 127.0f, kHi = kRoundMagic + 127.0f;
constexpr uint32_t kLo2 = 0xFF81FF81u, kHi2 = 0x007F007Fu;

// r = 1/s to within one ulp (rcp.approx; a subnormal s is flushed to 0 and
// gives r = inf, which sends the row to the exact path).  The fast codes'
// tie test flags every element within |y| 2^-21 + 2^-22 of a half-integer
// and so allows v r to be off the exact quotient by up to 2^-21 |y|: an
// exactly rounded r needs 2^-23 |y| (its own rounding and the quotient's),
// one ulp more 1.5 2^-23 |y|, still inside.  The codes stay exact.
__device__ __forceinline__ float approx_rcp(float s) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
    return r;
}

// Codes of 8 scaled elements at scale s (r ~ 1/s, see approx_rcp): packed
// fast path, then the exact quotient for any element near a rounding tie
// (rare).
// IN_RANGE: s and r come from this row's own abs-max am (s = am / 127,
// r ~ 1 / s finite, so s is normal), so no code needs the clamp: every
// |v| r <= am r < 127 (1 + 2^-24)(1 + 2^-23)^2 < 127.5, so rint(v r) is
// within [-127, 127].
template <bool IN_RANGE>
__device__ __forceinline__ uint2 fast_codes_tied(const float (&v)[8], float s, float r, bool narrow,
                                                 float tie_bound) {
    const float4 a = make_float4(v[0], v[1], v[2], v[3]), b = make_float4(v[4], v[5], v[6], v[7]);
    float dmax = 0.0f;
    uint2 code = IN_RANGE ? fast_codes8<true, false>(a, b, r, kLo, kHi, kLo2, kHi2, dmax)
                 : narrow ? fast_codes8<true>(a, b, r, kLo, kHi, kLo2, kHi2, dmax)
                          : fast_codes8<false>(a, b, r, kLo, kHi, kLo2, kHi2, dmax);
    if (dmax >= tie_bound) {
#pragma unroll  // unrolled: v stays in registers
        for (int i = 0; i < 8; ++i) {
            const float t = fmaf(v[i], r, kRoundMagic);
            const float rq = t - kRoundMagic;
            const float d = fmaf(v[i], r, -rq);
            if (fabsf(d) + fmaf(fabsf(rq), 4.76837158203125e-07f, 2.384185791015625e-07f) >= 0.5f) {
                const uint32_t qe = (uint32_t)exact_code(v[i], s, 127.0f) & 0xffu;
                const int sh = 8 * (i & 3);
                uint32_t &w = i < 4 ? code.x : code.y;
                w = (w & ~(0xffu << sh)) | (qe << sh);
            }
        }
    }
    return code;
}

// ROWS token rows per CTA iteration, all loaded before the first reduction.
// Measured on B200: one row per small CTA (32 elements per thread) with many
// CTAs per SM beats several rows per larger CTA and beats staging rows in
// shared memory with bulk copies.  The CTAs are persistent (as many as fit
// on the SMs at once) and software-pipelined: the loads of a CTA's next row
// are issued before the current row's reduction, so that two rows per CTA
// are in flight while one is quantized.
//
// STATIC: one scale for the whole tensor, S = range[0] / 127 (a range
// calibrated beforehand, see sq_static_range_update); no per-row reduction,
// values beyond the range saturate, and scale[row] (if given) receives S so
// that the GEMM's per-token dequant applies it unchanged.
//
// rowsum (nullable): R[row] = sum of the row's codes (exact), which the GEMM
// with asymmetric weights needs.
template <typename T, int E, int ROWS, bool STATIC>
__global__ void __launch_bounds__(512)
quant_act_kernel(const T *__restrict__ x, int64_t M, int64_t K, const float *__restrict__ inv_s,
                 const float *__restrict__ range, int8_t *__restrict__ q, float *__restrict__ scale,
                 int32_t *__restrict__ rowsum) {
    constexpr int C = E / 8;  // chunks per thread
    // inv_s is kept in registers across rows unless that would spill
    constexpr bool kCacheInvS = C * ROWS <= 4;
    __shared__ float red[2][ROWS][32];
    __shared__ int rsum_red[2][ROWS][32];
    const int T_ = blockDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = T_ >> 5;
    pdl_wait();     // x, inv_s and the outputs may belong to the previous kernel
    pdl_trigger();  // the GEMM that follows may launch (it waits for this grid)

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
    // x * inv_s of chunk c (inv_s from registers or from L1)
    auto scaled = [&](const Raw8<T> &raw, int c, float (&v)[8]) {
        raw.widen(v);
        if (inv_s) {
            if (!kCacheInvS) load8_f32(inv_s + ((int64_t)c * T_ + threadIdx.x) * 8, f[0]);
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = v[i] * f[kCacheInvS ? c : 0][i];
        }
    };

    auto load_rows = [&](Raw8<T> (&dst)[ROWS][C], int64_t r0) {
#pragma unroll
        for (int rr = 0; rr < ROWS; ++rr) {
#pragma unroll
            for (int c = 0; c < C; ++c) {
                if (live[c] && r0 + rr < M &&
                    dbg_index_ok(((int64_t)c * T_ + threadIdx.x) * 8 + 8 <= K))
                    dst[rr][c].load(x + (r0 + rr) * K + ((int64_t)c * T_ + threadIdx.x) * 8);
                else
                    dst[rr][c].zero();
            }
        }
    };
    const int64_t rstride = (int64_t)gridDim.x * ROWS;
    int parity = 0;
    Raw8<T> raw[ROWS][C];
    if ((int64_t)blockIdx.x * ROWS < M) load_rows(raw, (int64_t)blockIdx.x * ROWS);
    for (int64_t row0 = (int64_t)blockIdx.x * ROWS; row0 < M; row0 += rstride, parity ^= 1) {
        float amax[ROWS];  // dynamic: the row's abs-max; static: this thread's
        float v[ROWS][C][8];  // x * inv_s of these rows, kept for the codes
#pragma unroll
        for (int rr = 0; rr < ROWS; ++rr) {
            amax[rr] = 0.0f;
#pragma unroll
            for (int c = 0; c < C; ++c) {
#ifdef W8A8_DEBUG
                raw[rr][c].widen(v[rr][c]);
                dbg_check8(v[rr][c]);  // the input itself (zeros past the row)
#endif
                scaled(raw[rr][c], c, v[rr][c]);
#pragma unroll
                for (int i = 0; i < 8; i += 2) amax[rr] = fmax3(amax[rr], fabsf(v[rr][c][i]), fabsf(v[rr][c][i + 1]));
            }
            if (!STATIC) {
                amax[rr] = warp_max(amax[rr]);
                if (nwarps > 1 && lane == 0) red[parity][rr][warp] = amax[rr];
            }
        }
        // these rows now live in v: the registers take the CTA's next rows,
        // which load while these are reduced and quantized
        load_rows(raw, row0 + rstride);
        if (!STATIC && nwarps > 1) __syncthreads();  // red[parity] complete; red[parity^1] free for the next rows
#pragma unroll
        for (int rr = 0; rr < ROWS; ++rr) {
            const int64_t row = row0 + rr;
            if (row >= M) break;
            float am = amax[rr], s;
            if (STATIC) {
                s = __fdiv_rn(__ldg(range), 127.0f);
                if (scale && threadIdx.x == 0) scale[row] = s;
            } else {
                if (nwarps > 1) {  // (one warp: its butterfly already holds the row's abs-max)
                    am = red[parity][rr][0];
                    for (int w = 1; w < nwarps; ++w) am = fmaxf(am, red[parity][rr][w]);
                }
                s = __fdiv_rn(am, 127.0f);
                if (threadIdx.x == 0) scale[row] = s;
            }
            const float r = approx_rcp(s);
            const bool exact_only = !(fabsf(r) <= 3.402823466e38f);  // 1/s overflowed (or s == 0)
            // |v r| <= am r (about 127 in the dynamic case): below 2^14 the
            // int16 clamp of fast_codes8 applies; a fast code can differ from
            // the exact one only where |d| comes within |y| 2^-21 + 2^-22 of
            // 0.5 (in the static case am is this thread's abs-max)
            const bool narrow = am * r < 16384.0f;
            const float tie_bound = 0.5f - fmaf(am * r, 4.76837158203125e-07f, 2.384185791015625e-07f);
            int8_t *qr = q + row * K;
            int rsum = 0;
            if (s != 0.0f && !exact_only) {  // the usual row: fast codes
#pragma unroll
                for (int c = 0; c < C; ++c) {
                    if (!live[c]) continue;
                    const uint2 code = fast_codes_tied<!STATIC>(v[rr][c], s, r, narrow, tie_bound);
                    *reinterpret_cast<uint2 *>(qr + ((int64_t)c * T_ + threadIdx.x) * 8) = code;
                    if (rowsum) rsum = __dp4a((int)code.y, 0x01010101, __dp4a((int)code.x, 0x01010101, rsum));
                }
            } else {  // an all-zero row (every code 0), or 1/s not finite: exact quotients
#pragma unroll
                for (int c = 0; c < C; ++c) {
                    if (!live[c]) continue;
                    uint2 code = make_uint2(0u, 0u);
                    if (s != 0.0f) {
                        int e[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) e[i] = (int)sym_code(v[rr][c][i], s, r, 127.0f, true);
                        code = pack8_codes(e);
                    }
                    *reinterpret_cast<uint2 *>(qr + ((int64_t)c * T_ + threadIdx.x) * 8) = code;
                    if (rowsum) rsum = __dp4a((int)code.y, 0x01010101, __dp4a((int)code.x, 0x01010101, rsum));
                }
            }
            if (rowsum) {  // uniform: every thread of the CTA takes this branch
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) rsum += __shfl_xor_sync(0xffffffffu, rsum, o);
                if (nwarps == 1) {
                    if (lane == 0) rowsum[row] = rsum;
                } else {
                    if (lane == 0) rsum_red[parity][rr][warp] = rsum;
                    __syncthreads();
                    if (threadIdx.x == 0) {
                        int t = 0;
                        for (int w = 0; w < nwarps; ++w) t += rsum_red[parity][rr][w];
                        rowsum[row] = t;
                    }
                }
            }
        }
    }
}

template <typename T, int E, int ROWS, bool STATIC>
static void launch_quant_act(const void *x, int64_t M, int64_t K, const float *inv_s, const float *range,
                             int8_t *q, float *scale, int32_t *rowsum, int sms, cudaStream_t st) {
    int threads = (int)ceil_div(ceil_div(K, E), 32) * 32;
    // persistent: as many CTAs as fit on the SMs at once, each striding over
    // groups of ROWS rows
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_act_kernel<T, E, ROWS, STATIC>, threads, 0);
    per_sm = std::max(1, std::min(per_sm, 2048 / threads));
    int64_t grid = std::min<int64_t>(ceil_div(M, ROWS), (int64_t)sms * per_sm);
    launch_pdl(quant_act_kernel<T, E, ROWS, STATIC>, dim3((unsigned)grid), dim3(threads), 0, st, (const T *)x, M, K,
               inv_s, range, q, scale, rowsum);
}

// ------------------------------------------------ LayerNorm fused with step 4
// Persistent CTAs of T threads, one row at a time; thread t owns the E (8 or
// 16) contiguous columns [t E, t E + E), so its gamma, beta and inv_s stay in
// registers for every row, and the next row's loads are issued before the
// current row's reductions.  The row statistics are fp64 pairwise sums: the
// tree that halves the row padded with zeros to a power of two
// (S(lo, len) = S(lo, len/2) + S(lo + len/2, len/2)), so they do not depend on
// how the work is split.  A thread sums its 8-column chunks as subtrees of 8
// and combines them pairwise; the xor butterfly of a warp combines
// neighbouring threads' subtrees (a + b == b + a exactly, so every lane ends
// with the same sum), and one more butterfly over the warps' sums finishes
// the tree (T and E are powers of two).  Then mean = S / K,
// var = S(d^2) / K with d = h - mean, rstd = 1 / sqrt(var + eps) (IEEE fp64);
// m and r rounded to fp32, then per element y = ((h - m) r) gamma + beta and
// x' = y inv_s in fp32 with no fused multiply-add (the build contracts
// nothing), the row abs-max and the packed per-token codes.  X' never goes to
// memory.

// Pairwise sum of 8 values (a subtree of 8 leaves).
__device__ __forceinline__ double tree8(const double (&a)[8]) {
    return ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
}

// The thread subtrees of the whole CTA combined in tree order: warp
// butterfly, then a butterfly over the nwarps (a power of two) warp sums.
// red: this reduction's slot array; a slot is reused two rows later, after
// other barriers, so one barrier per reduction suffices.
__device__ __forceinline__ double block_tree_sum(double v, double *red, int lane, int warp, int nwarps) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = lane < nwarps ? red[lane] : 0.0;
    for (int o = 1; o < nwarps; o <<= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    return __shfl_sync(0xffffffffu, t, 0);
}

template <typename T, int E>
__global__ void __launch_bounds__(1024)
ln_quant_kernel(const T *__restrict__ h, int64_t M, int64_t K, const float *__restrict__ gamma,
                const float *__restrict__ beta, float eps, const float *__restrict__ inv_s, int8_t *__restrict__ q,
                float *__restrict__ scale) {
    constexpr int C = E / 8;
    __shared__ double redd[2][2][32];  // [row parity][mean, variance][warp]
    __shared__ float redf[2][32];      // [row parity][warp]: abs-max
    const int T_ = blockDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = T_ >> 5;
    const int64_t base = (int64_t)threadIdx.x * E;  // this thread's first column
    pdl_wait();     // h, gamma, beta, inv_s and the outputs may belong to the previous kernel
    pdl_trigger();  // the GEMM that follows may launch (it waits for this grid)
    bool live[C];  // K is a multiple of 8: a chunk is wholly inside the row or wholly past it
    float g[C][8], bt[C][8], f[C][8];
#pragma unroll
    for (int c = 0; c < C; ++c) {
        live[c] = base + 8 * c < K;
        const int64_t j = base + 8 * c;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            g[c][i] = 1.0f;
            bt[c][i] = 0.0f;
            f[c][i] = 1.0f;
        }
        if (live[c]) {
            if (gamma) load8_f32(gamma + j, g[c]);
            if (beta) load8_f32(beta + j, bt[c]);
            if (inv_s) load8_f32(inv_s + j, f[c]);
        }
    }
    const double kd = (double)K;
    // S / K: a power-of-two K scales exactly (the same correctly rounded value
    // as the division), any other K divides
    const bool k_pow2 = (K & (K - 1)) == 0;
    const double inv_kd = 1.0 / kd;
    auto over_k = [&](double sum) { return k_pow2 ? sum * inv_kd : sum / kd; };
    auto load_row = [&](Raw8<T> (&dst)[C], int64_t r) {
#pragma unroll
        for (int c = 0; c < C; ++c) {
            if (live[c] && r < M && dbg_index_ok(base + 8 * c + 8 <= K)) dst[c].load(h + r * K + base + 8 * c);
            else dst[c].zero();
        }
    };

    Raw8<T> raw[C];
    load_row(raw, blockIdx.x);
    int par = 0;
    for (int64_t row = blockIdx.x; row < M; row += gridDim.x, par ^= 1) {
        Raw8<T> nxt[C];
        load_row(nxt, row + gridDim.x);
        double part[C];
#pragma unroll
        for (int c = 0; c < C; ++c) {
            float v[8];
            raw[c].widen(v);  // zeros past the row
            dbg_check8(v);
            double a[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) a[i] = (double)v[i];
            part[c] = tree8(a);
        }
        double tsum = part[0];
        if (C == 2) tsum = part[0] + part[C - 1];
        const double mu = over_k(block_tree_sum(tsum, redd[par][0], lane, warp, nwarps));
#pragma unroll
        for (int c = 0; c < C; ++c) {
            float v[8];
            raw[c].widen(v);
            double a[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const double d = (double)v[i] - mu;
                a[i] = live[c] ? d * d : 0.0;  // the padding adds zeros, not (0 - mu)^2
            }
            part[c] = tree8(a);
        }
        tsum = part[0];
        if (C == 2) tsum = part[0] + part[C - 1];
        const double var = over_k(block_tree_sum(tsum, redd[par][1], lane, warp, nwarps));
        const double rstd = 1.0 / sqrt(var + (double)eps);
        const float m32 = (float)mu, r32 = (float)rstd;
        // x' = ((h - m) r) gamma + beta, times inv_s, each op in fp32
        float x[C][8];
        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            float v[8];
            raw[c].widen(v);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float n = __fmul_rn(__fsub_rn(v[i], m32), r32);
                const float y = __fadd_rn(__fmul_rn(n, g[c][i]), bt[c][i]);
                x[c][i] = __fmul_rn(y, f[c][i]);
                if (live[c]) amax = fmaxf(amax, fabsf(x[c][i]));
            }
        }
        amax = warp_max(amax);
        if (lane == 0) redf[par][warp] = amax;
        __syncthreads();
        const float am = warp_max(lane < nwarps ? redf[par][lane] : 0.0f);
        const float s = __fdiv_rn(am, 127.0f);
        if (threadIdx.x == 0) scale[row] = s;
        const float r = approx_rcp(s);
        const bool exact_only = !(fabsf(r) <= 3.402823466e38f);
        const bool narrow = am * r < 16384.0f;
        const float tie_bound = 0.5f - fmaf(am * r, 4.76837158203125e-07f, 2.384185791015625e-07f);
#pragma unroll
        for (int c = 0; c < C; ++c) {
            if (!live[c]) continue;
            uint2 code = make_uint2(0u, 0u);
            if (s == 0.0f) {
            } else if (exact_only) {
                int e[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) e[i] = (int)sym_code(x[c][i], s, r, 127.0f, true);
                code = pack8_codes(e);
            } else {
                code = fast_codes_tied<true>(x[c], s, r, narrow, tie_bound);
            }
            *reinterpret_cast<uint2 *>(q + row * K + base + 8 * c) = code;
        }
#pragma unroll
        for (int c = 0; c < C; ++c) raw[c] = nxt[c];
    }
}

// T threads of E contiguous columns each, T * E the power of two at or above
// K (at least one warp): E = 8 up to K = 8192 (T <= 1024), 16 above
// (K <= 16384).  Persistent: as many CTAs as fit on the SMs at once.
template <typename T, int E>
static void launch_ln_quant(const void *h, int64_t M, int64_t K, const float *gamma, const float *beta, float eps,
                            const float *inv_s, int8_t *q, float *scale, int sms, cudaStream_t st) {
    int64_t P = 32 * E;
    while (P < K) P *= 2;
    const int threads = (int)(P / E);
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ln_quant_kernel<T, E>, threads, 0);
    per_sm = std::max(1, std::min(per_sm, 2048 / threads));
    const int64_t grid = std::min<int64_t>(M, (int64_t)sms * per_sm);
    launch_pdl(ln_quant_kernel<T, E>, dim3((unsigned)grid), dim3(threads), 0, st, (const T *)h, M, K, gamma, beta, eps,
               inv_s, q, scale);
}

// E elements per thread: one warp per row up to K = 1024, then 32 elements
// per thread (measured faster than 64 at K = 4096: fewer registers, more
// rows in flight per SM), 64 past K = 16384 (at most 512 threads a row).
template <bool STATIC>
static void dispatch_quant(const void *x, bool bf, int64_t M, int64_t K, const float *inv_s, const float *range,
                           int8_t *q, float *scale, int32_t *rowsum, int sms, cudaStream_t cs) {
    if (K <= 256) {
        if (bf) launch_quant_act<__nv_bfloat16, 8, 1, STATIC>(x, M, K, inv_s, range, q, scale, rowsum, sms, cs);
        else launch_quant_act<float, 8, 1, STATIC>(x, M, K, inv_s, range, q, scale, rowsum, sms, cs);
    } else if (K <= 512) {
        if (bf) launch_quant_act<__nv_bfloat16, 16, 1, STATIC>(x, M, K, inv_s, range, q, scale, rowsum, sms, cs);
        else launch_quant_act<float, 16, 1, STATIC>(x, M, K, inv_s, range, q, scale, rowsum, sms, cs);
    } else if (K <= 1024) {
        if (bf) launch_quant_act<__nv_bfloat16, 32, 1, STATIC>(x, M, K, inv_s, range, q, scale, rowsum, sms, cs);
        else launch_quant_act<float, 32, 1, STATIC>(x, M, K, inv_s, range, q, scale, rowsum, sms, cs);
    } else if (K <= 16384) {
        if (bf) launch_quant_act<__nv_bfloat16, 32, 1, STATIC>(x, M, K, inv_s, range, q, scale, rowsum, sms, cs);
        else launch_quant_act<float, 32, 1, STATIC>(x, M, K, inv_s, range, q, scale, rowsum, sms, cs);
    } else {  // at most 512 threads a row
        if (bf) launch_quant_act<__nv_bfloat16, 64, 1, STATIC>(x, M, K, inv_s, range, q, scale, rowsum, sms, cs);
        else launch_quant_act<float, 64, 1, STATIC>(x, M, K, inv_s, range, q, scale, rowsum, sms, cs);
    }
}

// range = first ? a : fl(fl(rate range) + fl(fl(1 - rate) a)) with
// a = max_j fl(ax_j inv_s_j) -- the batch's abs-max of x * inv_s, since
// |x| c is monotonic in |x| for c >= 0.  One CTA.
__global__ void __launch_bounds__(1024)
static_range_kernel(const float *__restrict__ ax, const float *__restrict__ inv_s, int64_t K, float rate,
                    int first, float *__restrict__ range) {
    __shared__ float red[32];
    float a = 0.0f;
    for (int64_t j = threadIdx.x; j < K; j += blockDim.x) {
        const float v = inv_s ? __fmul_rn(ax[j], inv_s[j]) : ax[j];
        a = fmaxf(a, fabsf(v));
    }
    a = warp_max(a);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) a = fmaxf(a, red[w]);
        a = fmaxf(a, red[0]);
        range[0] = first ? a : __fadd_rn(__fmul_rn(rate, range[0]), __fmul_rn(__fsub_rn(1.0f, rate), a));
    }
}

W8A8_DEBUG_READER(quant_act)

}  // namespace w8a8

using namespace w8a8;

extern "C" sq_status quant_act_per_token(const void *x, sq_dtype xt, int64_t M, int64_t K,
                                         const float *inv_s, int8_t *q_out, float *scale_out,
                                         void *stream) {
    return quant_act_per_token_rowsum(x, xt, M, K, inv_s, q_out, scale_out, nullptr, stream);
}

extern "C" sq_status quant_act_per_token_rowsum(const void *x, sq_dtype xt, int64_t M, int64_t K,
                                                const float *inv_s, int8_t *q_out, float *scale_out,
                                                int32_t *rowsum_out, void *stream) {
    if (M > 0 && (!x || !q_out || !scale_out)) return fail(SQ_ERR_NULL, "quant_act_per_token: NULL pointer");
    if (rowsum_out && !aligned(rowsum_out, 4))
        return fail(SQ_ERR_ALIGN, "quant_act_per_token: misaligned rowsum_out");
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
    dispatch_quant<false>(x, xt == SQ_BF16, M, K, inv_s, nullptr, q_out, scale_out, rowsum_out, sms, cs);
    return launch_status("quant_act_kernel");
}

extern "C" sq_status sq_static_range_update(const float *x_absmax, const float *inv_s, int64_t K, float rate,
                                            int first, float *range, void *stream) {
    if (!x_absmax || !range) return fail(SQ_ERR_NULL, "sq_static_range_update: NULL pointer");
    if (K <= 0) return fail(SQ_ERR_SHAPE, "sq_static_range_update: K=%lld", (long long)K);
    if (!(rate >= 0.0f && rate <= 1.0f))
        return fail(SQ_ERR_ARG, "sq_static_range_update: rate=%g outside [0,1]", (double)rate);
    if (!aligned(x_absmax, 4) || !aligned(range, 4) || (inv_s && !aligned(inv_s, 4)))
        return fail(SQ_ERR_ALIGN, "sq_static_range_update: misaligned pointer");
    int sms;
    sq_status st = check_device(&sms);
    if (st != SQ_OK) return st;
    static_range_kernel<<<1, 1024, 0, (cudaStream_t)stream>>>(x_absmax, inv_s, K, rate, first != 0, range);
    return launch_status("static_range_kernel");
}

extern "C" sq_status quant_act_static(const void *x, sq_dtype xt, int64_t M, int64_t K, const float *inv_s,
                                      const float *range, int8_t *q_out, float *scale_out, int32_t *rowsum_out,
                                      void *stream) {
    if (M > 0 && (!x || !q_out || !range)) return fail(SQ_ERR_NULL, "quant_act_static: NULL pointer");
    if (xt != SQ_F32 && xt != SQ_BF16) return fail(SQ_ERR_DTYPE, "quant_act_static: dtype %d", (int)xt);
    if (M < 0 || K <= 0 || K % 16 != 0 || K > 32768)
        return fail(SQ_ERR_SHAPE, "quant_act_static: M=%lld K=%lld (K must be a multiple of 16 in [16, 32768])",
                    (long long)M, (long long)K);
    if (M == 0) return SQ_OK;
    if (!aligned(x, 16) || !aligned(q_out, 16) || !aligned(range, 4) || (scale_out && !aligned(scale_out, 4)) ||
        (inv_s && !aligned(inv_s, 16)) || (rowsum_out && !aligned(rowsum_out, 4)))
        return fail(SQ_ERR_ALIGN, "quant_act_static: misaligned pointer (x, q_out, inv_s need 16 bytes)");
    int sms;
    sq_status st = check_device(&sms);
    if (st != SQ_OK) return st;
    dispatch_quant<true>(x, xt == SQ_BF16, M, K, inv_s, range, q_out, scale_out, rowsum_out, sms,
                         (cudaStream_t)stream);
    return launch_status("quant_act_kernel");
}

extern "C" sq_status sq_layernorm_quant(const void *h, sq_dtype ht, int64_t M, int64_t K, const float *gamma,
                                        const float *beta, float eps, const float *inv_s, int8_t *q_out,
                                        float *scale_out, void *stream) {
    if (M > 0 && (!h || !q_out || !scale_out)) return fail(SQ_ERR_NULL, "sq_layernorm_quant: NULL pointer");
    if (ht != SQ_F32 && ht != SQ_BF16) return fail(SQ_ERR_DTYPE, "sq_layernorm_quant: dtype %d", (int)ht);
    if (M < 0 || K <= 0 || K % 16 != 0 || K > 16384)
        return fail(SQ_ERR_SHAPE, "sq_layernorm_quant: M=%lld K=%lld (K must be a multiple of 16 in [16, 16384])",
                    (long long)M, (long long)K);
    if (!(eps >= 0.0f) || isinf(eps)) return fail(SQ_ERR_ARG, "sq_layernorm_quant: eps=%g", (double)eps);
    if (M == 0) return SQ_OK;
    if (!aligned(h, 16) || !aligned(q_out, 16) || !aligned(scale_out, 4) || (gamma && !aligned(gamma, 16)) ||
        (beta && !aligned(beta, 16)) || (inv_s && !aligned(inv_s, 16)))
        return fail(SQ_ERR_ALIGN, "sq_layernorm_quant: misaligned pointer (h, q_out, gamma, beta, inv_s need 16 bytes)");
    int sms;
    sq_status st = check_device(&sms);
    if (st != SQ_OK) return st;
    cudaStream_t cs = (cudaStream_t)stream;
    const bool bf = ht == SQ_BF16;
    if (K <= 8192) {
        if (bf) launch_ln_quant<__nv_bfloat16, 8>(h, M, K, gamma, beta, eps, inv_s, q_out, scale_out, sms, cs);
        else launch_ln_quant<float, 8>(h, M, K, gamma, beta, eps, inv_s, q_out, scale_out, sms, cs);
    } else {
        if (bf) launch_ln_quant<__nv_bfloat16, 16>(h, M, K, gamma, beta, eps, inv_s, q_out, scale_out, sms, cs);
        else launch_ln_quant<float, 16>(h, M, K, gamma, beta, eps, inv_s, q_out, scale_out, sms, cs);
    }
    return launch_status("ln_quant_kernel");
}
