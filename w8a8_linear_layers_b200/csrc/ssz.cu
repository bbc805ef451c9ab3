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
// Readings (shared with the CPU oracle): the error of a scale c is the mean
// over K of (w - c Q(w,c))^2 after re-quantising at c; the relative and
// absolute tests are OR-ed, taken before the greedy update, and a channel
// stops for good once it meets them; the minimum scale floors the MinMax
// scale and every candidate; int4 codes are [-7, 7].
//
// Design.  One CTA of R warps per output channel; the row stays resident in
// shared memory for the whole search (W is read from HBM once, the codes
// written once), next to two code buffers: a round writes the candidate's
// codes into one while the kept codes stay in the other, and a kept
// candidate swaps them (the moved chunks' change of NUM and DEN reads both,
// with no code computed twice).  A bf16 row is kept as loaded (2 bytes an
// element) and folded again, fl(w s_j) with the same single fp32 rounding,
// wherever it is read (s through L1); an fp32 row is kept folded.  At
// K = 4096 a channel takes 16 KB.
//
// The error is evaluated exactly instead of by a per-element fp64 sum:
//     K e(c) = W2 - 2 c NUM + c^2 DEN,  W2 = sum w^2, NUM = sum w q, DEN = sum q^2,
// with W2 and NUM held in double-double (error-free transformations: Knuth's
// TwoSum and the FMA TwoProduct), DEN exact, and the cancelling sum taken
// with TwoSum.  NUM and DEN change only where a code changes, so a round is
// one pass that computes the codes at the candidate scale on the FP32 pipe
// (magic-constant rounding), compares them 8 at a time with the kept codes
// and updates NUM/DEN for the few that moved: DEN exactly, NUM by the exact
// products w (q' - q) summed in fp64 (a handful of terms per thread and
// round, each sum off by at most 2^-52 of the terms' magnitudes) and added
// to the double-double NUM with TwoSum.  The evaluated error is then within
// a few 2^-52 of |w| c per moved code of the exact one, far below the 1e-10
// thresholds the decisions test.
// Codes are exact: an element whose scaled value lies within |y| 2^-21 of a
// half-integer takes the IEEE quotient (see sym_code_i for the bound).
//
// The search is a chain of rounds per channel, so the kernel is latency
// bound; it keeps many channels in flight (small CTAs, shared-memory rows)
// and keeps each round's serial tail short: warp trees skip warps whose
// codes did not move, and with four or more warps a channel warp 0 alone
// takes the decision (the exact error in fp64 and the next candidate) and
// shares it through shared memory, so the other warps skip that fp64 work.
#include "common.cuh"
#include "dd.cuh"

namespace w8a8 {

constexpr double kSszThreshold = 1e-10;
constexpr float kSszMinScale = 1e-5f;

// K e(c) = W2 - 2 c NUM + c^2 DEN, exact up to one final rounding.  The
// search compares these K-scaled errors directly (K > 0 cancels), and
// divides by K only for the reported error.
__device__ __forceinline__ double exact_error_k(dd W2, dd NUM, int den, float c) {
    const double c2x = 2.0 * (double)c;               // exact
    const double p1 = c2x * NUM.hi;                   // 2 c NUM.hi = p1 + e1 exactly
    const double e1 = fma(c2x, NUM.hi, -p1);
    const double cc = (double)c * (double)c;           // exact (24-bit x 24-bit)
    const double dend = (double)den;
    const double p2 = dend * cc;                       // c^2 DEN = p2 + e2 exactly
    const double e2 = fma(dend, cc, -p2);
    const dd s1 = two_sum(W2.hi, -p1);
    const dd s2 = two_sum(s1.hi, p2);
    const double tail = ((s1.lo + s2.lo) + (W2.lo - e1)) + (e2 - c2x * NUM.lo);
    const double v = s2.hi + tail;
    // below the evaluation error (a few 2^-100 W2) the error is zero
    return fabs(v) <= W2.hi * 0x1p-96 ? 0.0 : v;
}

// Next least-squares candidate from the kept sums (oracle: fp32 of the fp64
// quotient, floored at the minimum scale; no codes: keep the scale).
__device__ __forceinline__ float ls_candidate(dd NUM, int den, float keep) {
    return den != 0 ? fmaxf((float)((NUM.hi + NUM.lo) / (double)den), kSszMinScale) : keep;
}

__device__ __forceinline__ int code_byte(uint2 p, int b) {
    const uint32_t w = b < 4 ? p.x : p.y;
    return (int)(int8_t)((w >> (8 * (b & 3))) & 0xffu);
}

struct PassOut {
    dd num;          // init: NUM
    dd w2;           // init only
    double dnum;     // update: change of NUM (exact products, fp64 sum)
    int den;         // init: DEN; update: change of DEN
    bool moved;      // update: some code of this thread changed
};

// The channel's row in shared memory, read as folded fp32 values.  fp32
// input: the folded row itself.  bf16 input: the raw bf16 row, widened
// (exact) and, with FOLD, multiplied by s_j (one IEEE fp32 multiply, the
// value the fp32 path stores).
template <typename T, bool FOLD> struct Row;

template <bool FOLD> struct Row<float, FOLD> {
    const float *w;
    __device__ __forceinline__ void load8(int j, float4 &a, float4 &b) const {
        a = *reinterpret_cast<const float4 *>(w + j);
        b = *reinterpret_cast<const float4 *>(w + j + 4);
    }
    __device__ __forceinline__ float load1(int j) const { return w[j]; }
};

template <bool FOLD> struct Row<__nv_bfloat16, FOLD> {
    const uint16_t *w;     // raw bf16 bits
    const float *s;        // smoothing factor (global, read through L1); unused without FOLD
    __device__ __forceinline__ void load8(int j, float4 &a, float4 &b) const {
        const uint4 u = *reinterpret_cast<const uint4 *>(w + j);
        a = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                        __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
        b = make_float4(__uint_as_float(u.z << 16), __uint_as_float(u.z & 0xffff0000u),
                        __uint_as_float(u.w << 16), __uint_as_float(u.w & 0xffff0000u));
        if (FOLD) {
            const float4 f0 = __ldg(reinterpret_cast<const float4 *>(s + j));
            const float4 f1 = __ldg(reinterpret_cast<const float4 *>(s + j) + 1);
            a = make_float4(__fmul_rn(a.x, f0.x), __fmul_rn(a.y, f0.y), __fmul_rn(a.z, f0.z), __fmul_rn(a.w, f0.w));
            b = make_float4(__fmul_rn(b.x, f1.x), __fmul_rn(b.y, f1.y), __fmul_rn(b.z, f1.z), __fmul_rn(b.w, f1.w));
        }
    }
    __device__ __forceinline__ float load1(int j) const {
        const float v = __uint_as_float((uint32_t)w[j] << 16);
        return FOLD ? __fmul_rn(v, __ldg(s + j)) : v;
    }
    // the folded values of 8 raw elements u at column j (staging)
    __device__ __forceinline__ void load8_global(uint4 u, int j, float4 &a, float4 &b) const {
        a = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                        __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
        b = make_float4(__uint_as_float(u.z << 16), __uint_as_float(u.z & 0xffff0000u),
                        __uint_as_float(u.w << 16), __uint_as_float(u.w & 0xffff0000u));
        if (FOLD) {
            const float4 f0 = __ldg(reinterpret_cast<const float4 *>(s + j));
            const float4 f1 = __ldg(reinterpret_cast<const float4 *>(s + j) + 1);
            a = make_float4(__fmul_rn(a.x, f0.x), __fmul_rn(a.y, f0.y), __fmul_rn(a.z, f0.z), __fmul_rn(a.w, f0.w));
            b = make_float4(__fmul_rn(b.x, f1.x), __fmul_rn(b.y, f1.y), __fmul_rn(b.z, f1.z), __fmul_rn(b.w, f1.w));
        }
    }
};

// Main loop of a pass over this thread's chunks.  init: writes the codes
// into q and accumulates W2, NUM, DEN.  update: writes the codes at the
// candidate into qc, compares them with the kept codes in q and marks the
// chunks that moved; their change of NUM and DEN is taken afterwards, once
// (a warp would otherwise run that path whenever any lane had a moved
// chunk).  Both mark near-tie chunks.
template <bool INIT, bool NARROW, typename R>
__device__ __forceinline__ void pass_chunks(const R &row, int K, float r, float lo, float hi,
                                            uint32_t lo2, uint32_t hi2, float tie_bound, int8_t *__restrict__ q,
                                            int8_t *__restrict__ qc, PassOut &out, uint32_t &moved,
                                            uint32_t &tie) {
    const int stride = blockDim.x * 8;
    int m = 0;
#pragma unroll 2
    for (int j = threadIdx.x * 8; j < K; j += stride, ++m) {
        float dmax = 0.0f;
        float4 a, b;
        row.load8(j, a, b);
        const uint2 nw = fast_codes8<NARROW>(a, b, r, lo, hi, lo2, hi2, dmax);
        if (dmax >= tie_bound) tie |= 1u << m;
        if (INIT) {
            *reinterpret_cast<uint2 *>(q + j) = nw;
            const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int qq = code_byte(nw, i);
                const double wd = (double)v[i];
                dd_acc(out.w2, wd * wd);                // exact product
                dd_acc(out.num, wd * code_to_f64(qq));  // exact product
                out.den += qq * qq;
            }
        } else {
            *reinterpret_cast<uint2 *>(qc + j) = nw;
            const uint2 od = *reinterpret_cast<const uint2 *>(q + j);
            if ((nw.x ^ od.x) | (nw.y ^ od.y)) moved |= 1u << m;
        }
    }
}

// Moved chunks: the change of NUM and DEN from the kept codes (q) to the
// candidate's (qc).
// The change of DEN for a chunk whose codes go from od to nw (exact: dp4a
// of the signed bytes).
__device__ __forceinline__ int den_change(uint2 nw, uint2 od) {
    return __dp4a((int)nw.x, (int)nw.x, __dp4a((int)nw.y, (int)nw.y, 0)) -
           __dp4a((int)od.x, (int)od.x, __dp4a((int)od.y, (int)od.y, 0));
}

template <typename R>
__device__ __forceinline__ void sum_moved(const R &row, uint32_t moved, const int8_t *__restrict__ q,
                                          const int8_t *__restrict__ qc, PassOut &out) {
    const int stride = blockDim.x * 8;
    while (moved) {
        const int mm = __ffs(moved) - 1;
        moved &= moved - 1u;
        const int j = threadIdx.x * 8 + mm * stride;
        const uint2 nw = *reinterpret_cast<const uint2 *>(qc + j);
        const uint2 od = *reinterpret_cast<const uint2 *>(q + j);
        out.den += den_change(nw, od);
        // only the bytes that differ: 0x80 marks each
        const unsigned long long diff =
            ((unsigned long long)__vcmpne4(nw.y, od.y) << 32 | __vcmpne4(nw.x, od.x)) & 0x8080808080808080ull;
        for (unsigned long long d = diff; d;) {
            const int i = (__ffsll((long long)d) - 1) >> 3;
            d &= d - 1ull;
            out.dnum += (double)row.load1(j + i) * code_to_f64(code_byte(nw, i) - code_byte(od, i));  // exact product
        }
    }
}

// Near-tie chunks (rare): the exact quotient decides their flagged elements,
// whose fast codes are already in q.  With SUMS, the change of NUM and DEN
// is accumulated.  Visiting only the flagged chunks keeps the warp's detour
// short when one lane has a near tie.
// SUMS: 1 adds the change to the init sums (double-double NUM), 2 to the
// update's fp64 change of NUM, 0 to nothing.
template <int SUMS, typename R>
__device__ __forceinline__ void fix_ties(const R &row, uint32_t tie, float c, float r, float qmax,
                                         int8_t *__restrict__ q, PassOut &out) {
    const int stride = blockDim.x * 8;
    while (tie) {
        const int mm = __ffs(tie) - 1;
        tie &= tie - 1u;
        const int j = threadIdx.x * 8 + mm * stride;
#pragma unroll 1
        for (int i = 0; i < 8; ++i) {
            const float v = row.load1(j + i);
            const float t = fmaf(v, r, kRoundMagic);
            const float rq = t - kRoundMagic;
            const float d = fmaf(v, r, -rq);
            if (fabsf(d) + fmaf(fabsf(rq), 4.76837158203125e-07f, 2.384185791015625e-07f) >= 0.5f) {
                const int qf = (int)q[j + i];
                const int qe = exact_code(v, c, qmax);
                if (qe != qf) {
                    q[j + i] = (int8_t)qe;
                    if (SUMS) {
                        out.den += qe * qe - qf * qf;
                        if (SUMS == 1) dd_acc(out.num, (double)v * code_to_f64(qe - qf));
                        else out.dnum += (double)v * code_to_f64(qe - qf);
                        out.moved = true;
                    }
                }
            }
        }
    }
}

struct ScaleConsts {
    float r, lo, hi, tie_bound;
    uint32_t lo2, hi2;
    bool narrow;
};

// Per-scale constants of a pass; narrow is warp-uniform.  Called by whole warps.
__device__ __forceinline__ ScaleConsts scale_consts(float c, float qmax, float wmax) {
    ScaleConsts k;
    k.r = __fdiv_rn(1.0f, c);  // c >= 1e-5, so r is finite
    k.lo = kRoundMagic - qmax;
    k.hi = kRoundMagic + qmax;
    const uint32_t qm = (uint32_t)(int)qmax;
    k.hi2 = qm | (qm << 16);
    k.lo2 = ((0x10000u - qm) & 0xffffu) * 0x10001u;
    // a fast code can differ from the exact one only where |d| comes within
    // |y| 2^-21 + 2^-22 of 0.5, and |y| <= wmax r
    k.tie_bound = 0.5f - fmaf(wmax * k.r, 4.76837158203125e-07f, 2.384185791015625e-07f);
    k.narrow = __all_sync(0xffffffffu, wmax * k.r < 16384.0f);
    return k;
}

// One pass at scale c over this thread's chunks of the row in shared memory.
// init: q receives the codes at c and W2, NUM, DEN are accumulated.  update:
// qc receives the codes at c (q keeps the kept codes) and the change of NUM
// and DEN from q to qc is returned; if c is kept the caller swaps the two
// buffers, if not q still holds the kept codes.  wmax is the thread's max
// |w|.  Called by whole warps.
template <bool INIT, typename R>
__device__ __forceinline__ PassOut row_pass(const R &row, int K, float c, float qmax, float wmax,
                                            int8_t *__restrict__ q, int8_t *__restrict__ qc) {
    const ScaleConsts k = scale_consts(c, qmax, wmax);
    PassOut out = {{0.0, 0.0}, {0.0, 0.0}, 0.0, 0, false};
    uint32_t moved = 0u;  // bit m: chunk m of this thread moved (at most 32 chunks per thread)
    uint32_t tie = 0u;    // bit m: chunk m holds an element near a rounding tie
    if (k.narrow)
        pass_chunks<INIT, true>(row, K, k.r, k.lo, k.hi, k.lo2, k.hi2, k.tie_bound, q, qc, out, moved, tie);
    else
        pass_chunks<INIT, false>(row, K, k.r, k.lo, k.hi, k.lo2, k.hi2, k.tie_bound, q, qc, out, moved, tie);
    if (!INIT) {
        out.moved = moved != 0u;
        sum_moved(row, moved, q, qc, out);
    }
    fix_ties<INIT ? 1 : 2>(row, tie, c, k.r, qmax, INIT ? q : qc, out);
    return out;
}

struct WarpPart {
    dd num, w2;  // init: the warp's NUM and W2; update: num.hi is the warp's change of NUM
    int den;
};


// Dynamic shared memory: the row (K elements, bf16 raw or fp32 folded), two
// code buffers (K bytes each), then the per-warp partials of two rounds
// (8-byte aligned).
__host__ __device__ __forceinline__ size_t ssz_parts_offset(int K, size_t elem) {
    return ((size_t)K * elem + 2 * (size_t)K + 7) & ~(size_t)7;
}

template <typename T, bool FOLD>
__global__ void __launch_bounds__(512, 2)
ssz_kernel(const T *__restrict__ wg, int64_t N, int K, const float *__restrict__ s, float qmax, int max_iters,
           int8_t *__restrict__ q_out, float *__restrict__ scale_out, double *__restrict__ mse_out,
           int32_t *__restrict__ iters_out) {
    extern __shared__ __align__(16) uint8_t smem[];
    T *wrow = reinterpret_cast<T *>(smem);                     // K elements: the row (see Row)
    // two code buffers of K bytes: the kept codes (q) and a round's candidate
    // codes (qc), swapped when the candidate is kept; then the per-warp
    // partials of two rounds
    int8_t *q = reinterpret_cast<int8_t *>(smem) + (size_t)K * sizeof(T);
    int8_t *qc = q + K;
    WarpPart *parts = reinterpret_cast<WarpPart *>(smem + ssz_parts_offset(K, sizeof(T)));
    Row<T, FOLD> row;
    if constexpr (sizeof(T) == 2) {
        row.w = reinterpret_cast<const uint16_t *>(wrow);
        row.s = s;
    } else {
        row.w = reinterpret_cast<const float *>(wrow);
    }
    struct Decision {
        float c_next;
        int keep, done;
    };
    __shared__ Decision decision[2];  // warp 0's decision of a round, by parity
    __shared__ float redmax[16];
    const int T_ = blockDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = T_ >> 5;
    const double kd = (double)K;
    const double thr_k = kSszThreshold * kd;  // absolute threshold on K-scaled errors

    for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
        // ---- stage the row in shared memory (bf16 as loaded, fp32 folded)
        float amax = 0.0f;
#pragma unroll 4
        for (int j = threadIdx.x * 8; j < K; j += T_ * 8) {
            float v[8];
            if constexpr (sizeof(T) == 2) {
                const uint4 u = __ldg(reinterpret_cast<const uint4 *>(wg + n * K + j));
                *reinterpret_cast<uint4 *>(wrow + j) = u;
                float4 a, b;
                row.load8_global(u, j, a, b);
                v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
                v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
            } else {
                Vec8<T>::load(wg + n * K + j, v);
                if (FOLD) {
                    float f[8];
                    load8_f32(s + j, f);
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], f[i]);
                }
                float4 *dst = reinterpret_cast<float4 *>(wrow + j);
                dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                dst[1] = make_float4(v[4], v[5], v[6], v[7]);
            }
            dbg_check8(v);  // the (smoothed) weights the search reads
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
        }
        const float wmax = amax;  // this thread's max |w| (tie bound)
        amax = warp_max(amax);
        if (lane == 0) redmax[warp] = amax;
        __syncthreads();
        amax = redmax[0];
        for (int i = 1; i < nwarps; ++i) amax = fmaxf(amax, redmax[i]);

        // ---- MinMax init: codes into q, exact W2 / NUM / DEN
        float s_best = fmaxf(__fdiv_rn(amax, qmax), kSszMinScale);
        int par = 0;
        {
            PassOut p = row_pass<true>(row, K, s_best, qmax, wmax, q, qc);
            p.num = warp_sum_dd(p.num);
            p.w2 = warp_sum_dd(p.w2);
            p.den = warp_sum_i(p.den);
            if (lane == 0) parts[par * nwarps + warp] = {p.num, p.w2, p.den};
        }
        __syncthreads();
        // every thread holds the (identical) channel state
        dd W2 = parts[par * nwarps].w2, NUM = parts[par * nwarps].num;
        int DEN = parts[par * nwarps].den;
        for (int i = 1; i < nwarps; ++i) {
            W2 = dd_add_cascade(W2, parts[par * nwarps + i].w2);
            NUM = dd_add_cascade(NUM, parts[par * nwarps + i].num);
            DEN += parts[par * nwarps + i].den;
        }
        double m_best = exact_error_k(W2, NUM, DEN, s_best);  // K x error
        float c = ls_candidate(NUM, DEN, s_best);
        int it = 0;
        bool done = max_iters == 0;

        // ---- least-squares rounds.  A round writes its candidate codes into
        // qc; a kept candidate swaps the buffers, a rejected one (which ends
        // the search: its improvement is <= 0, below both thresholds) leaves
        // the kept codes in q.
        while (!done) {
            par ^= 1;
            PassOut p = row_pass<false>(row, K, c, qmax, wmax, q, qc);
            if (__any_sync(0xffffffffu, p.moved)) {
                p.dnum = warp_sum_d(p.dnum);
                p.den = warp_sum_i(p.den);
            } else {
                p.dnum = 0.0;
                p.den = 0;
            }
            if (lane == 0) parts[par * nwarps + warp] = {{p.dnum, 0.0}, {0.0, 0.0}, p.den};
            __syncthreads();  // the candidate codes and all partials are in place
            ++it;
            // The decision: every thread takes it (1-2 warps a channel), or
            // warp 0 takes it and shares it (4 or more warps, where the
            // saved fp64 work outweighs one more barrier; measured).
            const bool shared_decision = nwarps >= 4;
            if (!shared_decision || warp == 0) {
                dd num_c = NUM;
                int den_c = DEN;
                for (int i = 0; i < nwarps; ++i) {
                    dd_acc(num_c, parts[par * nwarps + i].num.hi);
                    den_c += parts[par * nwarps + i].den;
                }
                const double m_c = exact_error_k(W2, num_c, den_c, c);
                const float c_next = ls_candidate(num_c, den_c, c);  // used only if c is kept
                // on K-scaled errors: d/e < thr <=> dK < thr eK (eK > 0), |d| < thr <=> |dK| < thr K
                const double delta = m_best - m_c;
                bool dn = (m_best == 0.0) || (delta < kSszThreshold * m_best) || (fabs(delta) < thr_k) ||
                          it == max_iters;
                const bool keep = m_c < m_best;
                if (keep) {
                    m_best = m_c;
                    NUM = num_c;
                    DEN = den_c;
                } else {
                    dn = true;  // implied by the tests above (m_best >= 0); q keeps the kept codes
                }
                if (shared_decision) {
                    if (lane == 0) decision[par] = {c_next, keep ? 1 : 0, dn ? 1 : 0};
                } else {
                    done = dn;
                    if (keep) {
                        s_best = c;
                        c = c_next;
                        int8_t *t = q;  // the candidate's codes become the kept ones
                        q = qc;
                        qc = t;
                    }
                }
            }
            if (shared_decision) {
                __syncthreads();
                const Decision dcs = decision[par];
                done = dcs.done != 0;
                if (dcs.keep) {
                    s_best = c;
                    c = dcs.c_next;
                    int8_t *t = q;  // the candidate's codes become the kept ones
                    q = qc;
                    qc = t;
                }
            }
            // part[par] and decision[par] are rewritten two rounds from now,
            // after another barrier
        }

        // ---- kept codes out (each thread wrote and now reads its own chunks)
        for (int j = threadIdx.x * 8; j < K; j += T_ * 8)
            *reinterpret_cast<uint2 *>(q_out + n * K + j) = *reinterpret_cast<const uint2 *>(q + j);
        if (threadIdx.x == 0) {
            scale_out[n] = s_best;
            if (mse_out) mse_out[n] = m_best / kd;
            if (iters_out) iters_out[n] = it;
        }
        __syncthreads();  // shared row and buffers are reused by the next channel
    }
}

// Warps per channel: enough channels in flight per SM to cover each round's
// serial tail, enough warps per channel to spread a pass.
static int ssz_warps(int64_t K) {
#ifdef W8A8_SSZ_WARPS
    int64_t w = W8A8_SSZ_WARPS;
#else
    int64_t w = ceil_div(K, 2048);
#endif
    // at most 32 chunks of 8 per thread (the moved-chunk mask is 32 bits)
    w = std::max<int64_t>(w, ceil_div(K, 32 * 32 * 8));
    return (int)std::min<int64_t>(16, std::max<int64_t>(1, w));
}

template <typename T>
static sq_status launch_ssz(const void *w, int64_t N, int64_t K, const float *s, int bits, int max_iters,
                            int8_t *q, float *scale, double *mse, int32_t *iters, int sms, cudaStream_t st) {
    const int threads = 32 * ssz_warps(K);
    const float qmax = (float)((1 << (bits - 1)) - 1);
    const size_t smem = ssz_parts_offset((int)K, sizeof(T)) + sizeof(WarpPart) * 2 * (threads / 32);
    auto kern = s ? ssz_kernel<T, true> : ssz_kernel<T, false>;
    if (smem > 32 * 1024) {  // dynamic + static shared memory may pass the 48 KB default
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    }
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
    const int64_t grid = std::min<int64_t>(N, (int64_t)sms * std::max(per_sm, 1) * 8);
    kern<<<(unsigned)grid, threads, smem, st>>>((const T *)w, N, (int)K, s, qmax, max_iters, q, scale, mse, iters);
    return launch_status("ssz_kernel");
}

W8A8_DEBUG_READER(ssz)

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
    if (wt == SQ_BF16)
        return launch_ssz<__nv_bfloat16>(w, N, K, s, bits, max_iters, q_out, scale_out, mse_out, iters_out, sms, cs);
    return launch_ssz<float>(w, N, K, s, bits, max_iters, q_out, scale_out, mse_out, iters_out, sms, cs);
}
