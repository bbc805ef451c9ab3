// common.cuh -- helpers shared by the libw8a8 kernels and entry points.
//
// Device side: 16-byte vector loads of bf16/fp32 rows, warp/block
// reductions, and the exact symmetric quantizer.  Host side: argument
// checking, the thread-local error detail, device queries.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stdio.h>
#include <stdarg.h>

#include <algorithm>

#include "w8a8.h"

namespace w8a8 {

// ----------------------------------------------------------------- host side
void set_detail(const char *fmt, ...);

inline sq_status fail(sq_status s, const char *fmt, ...) {
    char buf[256];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    set_detail("%s", buf);
    return s;
}

// Compute capability 10.0 check for the current device; fills the SM count.
sq_status check_device(int *sm_count);

inline bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

inline sq_status launch_status(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return fail(SQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return SQ_OK;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ------------------------------------------------ programmatic dependent launch
// The per-inference kernels (activation quantization, GEMM) are launched with
// programmatic stream serialization: such a kernel may be scheduled before
// its predecessor in the stream has finished, as soon as every CTA of the
// predecessor has called pdl_trigger (or exited), so that its launch and
// prologue overlap the predecessor's tail.  Before its first access to global
// memory that the predecessor may write or read, every thread calls pdl_wait,
// which returns once the predecessor grid has completed and its writes are
// visible.  Without the attribute (or after a kernel that never triggers)
// both are no-ops and the launch is ordinary.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// ----------------------------------------------------------------- device side
// Load 8 consecutive elements (16 bytes of bf16, or 32 bytes of fp32) as fp32.
// bf16 widens exactly (its bits are the high half of an fp32).
template <typename T> struct Vec8;

template <> struct Vec8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&v)[8]) {
        uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

template <> struct Vec8<float> {
    static __device__ __forceinline__ void load(const float *p, float (&v)[8]) {
        float4 a = __ldg(reinterpret_cast<const float4 *>(p));
        float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

__device__ __forceinline__ void load8_f32(const float *p, float (&v)[8]) {
    Vec8<float>::load(p, v);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Symmetric code clamp(rint(v / s), -qmax, qmax) (round half to even),
// bit-identical to an IEEE fp32 division followed by rint, for qmax <= 127.
//
// Fast path, all on the FMA pipe: with r = RN(1/s) and the magic constant
// M = 1.5 * 2^23, t = fma(v, r, M) = RN(v r + M), which for |v r| < 2^22 is M
// plus v r rounded to an integer (ties to even; M is even) -- the EXACT
// product v r, rounded once.  Since r carries one rounding (2^-24 relative)
// and the IEEE quotient another, |v r - RN(v/s)| <= 2^-23 |y|, so the two
// round to the same integer unless a half-integer lies within 2^-23 |y|.
// d = fma(v, r, M - t) = RN(v r - rint(v r)) measures the distance to the
// nearest integer (M - t is exact); when |d| comes within
// |rint| 2^-21 + 2^-22 (>= 2^-21 |y|, a 4x margin) of 0.5 the exact quotient
// is taken.  Larger |v r| only ever clamps.  Returns the code as an int.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr int kRoundMagicBits = 0x4B400000;

__device__ __forceinline__ int sym_code_i(float v, float s, float r, float qmax) {
    float t = fmaf(v, r, kRoundMagic);
    const float rq = t - kRoundMagic;
    const float d = fmaf(v, r, -rq);
    if (fabsf(d) + fmaf(fabsf(rq), 4.76837158203125e-07f, 2.384185791015625e-07f) >= 0.5f)
        t = rintf(__fdiv_rn(v, s)) + kRoundMagic;  // near a tie: exact quotient
    t = fminf(fmaxf(t, kRoundMagic - qmax), kRoundMagic + qmax);
    return __float_as_int(t) - kRoundMagicBits;
}

// Same code as a float; `exact_only` forces the IEEE division (used when
// r = 1/s is not finite, i.e. s below ~2^-126).
__device__ __forceinline__ float sym_code(float v, float s, float r, float qmax, bool exact_only) {
    if (exact_only) return fminf(fmaxf(rintf(__fdiv_rn(v, s)), -qmax), qmax);
    return (float)sym_code_i(v, s, r, qmax);
}

// Exact fp64 value of a small integer code without a conversion instruction:
// the double with high word 0x43300000 and low word (q + 2^31) is
// 2^52 + 2^31 + q.
__device__ __forceinline__ double code_to_f64(int q) {
    return __hiloint2double(0x43300000, q ^ (int)0x80000000) - 4503601774854144.0;
}

// Packed two-lane fp32 arithmetic of sm_100 (fma/sub .rn.f32x2): each lane
// rounds exactly like the scalar IEEE operation.  Only fused multiply-adds
// and subtractions are used, so there is no separate product for the
// compiler to fuse with a later add.
union F2U {
    float2 f;
    unsigned long long u;
};

__device__ __forceinline__ float2 f2_fma(float2 a, float2 b, float2 c) {
    F2U x{a}, y{b}, z{c}, r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r.u) : "l"(x.u), "l"(y.u), "l"(z.u));
    return r.f;
}

__device__ __forceinline__ float2 f2_sub(float2 a, float2 b) {
    F2U x{a}, y{b}, r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r.u) : "l"(x.u), "l"(y.u));
    return r.f;
}

// Pack 8 integer codes in [-127,127] into 8 bytes.
__device__ __forceinline__ uint2 pack8_codes(const int (&q)[8]) {
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        lo |= ((uint32_t)q[i] & 0xffu) << (8 * i);
        hi |= ((uint32_t)q[4 + i] & 0xffu) << (8 * i);
    }
    return make_uint2(lo, hi);
}

// The exact code of one element (IEEE quotient), out of line: only taken for
// the rare elements near a rounding tie, so the division stays off the fast
// path (inlined, the compiler may predicate it onto every element).
static __device__ __noinline__ int exact_code(float v, float c, float qmax) {
    return (int)fminf(fmaxf(rintf(__fdiv_rn(v, c)), -qmax), qmax);
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ uint32_t clamp_s16x2(uint32_t w, uint32_t lo2, uint32_t hi2) {
    asm("max.s16x2 %0, %0, %1;" : "+r"(w) : "r"(lo2));
    asm("min.s16x2 %0, %0, %1;" : "+r"(w) : "r"(hi2));
    return w;
}

// Codes of 8 consecutive elements at scale c (fast path, see sym_code_i)
// packed in 8 bytes, two elements per instruction: t = fma(v, r, M) and
// d = fma(v, r, M - t).  dmax collects max |d| for the tie test.
// NARROW (every |v r| < 2^14): bits(t) - bits(M) is the code, so the low
// halves of bits(t) are the codes as int16 and are clamped two at a time;
// otherwise t is clamped as a float (|v r| may leave the integer range of M).
// !CLAMP: the caller guarantees every |v r| < qmax + 0.5, so rint(v r) is
// already in range and the low byte of bits(t) is the code as it stands.
template <bool NARROW, bool CLAMP = true>
__device__ __forceinline__ uint2 fast_codes8(const float4 a, const float4 b, float r, float lo, float hi,
                                             uint32_t lo2, uint32_t hi2, float &dmax) {
    const float2 v[4] = {make_float2(a.x, a.y), make_float2(a.z, a.w), make_float2(b.x, b.y), make_float2(b.z, b.w)};
    const float2 r2 = make_float2(r, r), m2 = make_float2(kRoundMagic, kRoundMagic);
    uint32_t t[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 tt = f2_fma(v[i], r2, m2);
        const float2 d = f2_fma(v[i], r2, f2_sub(m2, tt));
        dmax = fmax3(dmax, fabsf(d.x), fabsf(d.y));
        t[2 * i] = __float_as_uint(NARROW || !CLAMP ? tt.x : fminf(fmaxf(tt.x, lo), hi));  // code = low byte
        t[2 * i + 1] = __float_as_uint(NARROW || !CLAMP ? tt.y : fminf(fmaxf(tt.y, lo), hi));
    }
    if (NARROW && CLAMP) {
        uint32_t h[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = clamp_s16x2(__byte_perm(t[2 * i], t[2 * i + 1], 0x5410), lo2, hi2);
        return make_uint2(__byte_perm(h[0], h[1], 0x6420), __byte_perm(h[2], h[3], 0x6420));
    }
    const uint32_t p0 = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
    const uint32_t p1 = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410);
    return make_uint2(p0, p1);
}

// ------------------------------------------------------------ debug counters
// Debug builds (-DW8A8_DEBUG, libw8a8_debug.so): the kernels count the
// non-finite values they read from their inputs, and the index checks that
// fail (the access is then skipped), into two device counters per source
// file; sq_debug_status adds them up and clears them.  Nothing traps.  In
// release builds the checks compile to nothing.
#ifdef W8A8_DEBUG
static __device__ unsigned long long g_dbg_counts[2];  // [non-finite inputs, failed index checks]

__device__ __forceinline__ void dbg_count_nonfinite(int n) {
    if (n) atomicAdd(&g_dbg_counts[0], (unsigned long long)n);
}
__device__ __forceinline__ bool dbg_index_ok(bool ok) {
    if (!ok) atomicAdd(&g_dbg_counts[1], 1ull);
    return ok;
}
// reads and clears this source file's counters (host)
static inline cudaError_t dbg_take(cudaStream_t st, unsigned long long (&out)[2]) {
    unsigned long long zero[2] = {0ull, 0ull};
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_dbg_counts, sizeof out, 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_dbg_counts, zero, sizeof zero, 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return e;
}
// per-file readers (each file's counters are its own)
cudaError_t dbg_take_smooth(cudaStream_t st, unsigned long long (&out)[2]);
cudaError_t dbg_take_quant_act(cudaStream_t st, unsigned long long (&out)[2]);
cudaError_t dbg_take_ssz(cudaStream_t st, unsigned long long (&out)[2]);
cudaError_t dbg_take_ssz_asym(cudaStream_t st, unsigned long long (&out)[2]);
// the same check again, not counted (the paired use of a skipped access)
__device__ __forceinline__ bool dbg_index_again(bool ok) { return ok; }
#define W8A8_DEBUG_READER(name) \
    cudaError_t dbg_take_##name(cudaStream_t st, unsigned long long (&out)[2]) { return dbg_take(st, out); }
#else
__device__ __forceinline__ void dbg_count_nonfinite(int) {}
__device__ __forceinline__ bool dbg_index_ok(bool) { return true; }
__device__ __forceinline__ bool dbg_index_again(bool) { return true; }
#define W8A8_DEBUG_READER(name)
#endif

// Non-finite values among 8 (4) fp32 values (debug builds only).
__device__ __forceinline__ void dbg_check8(const float (&v)[8]) {
#ifdef W8A8_DEBUG
    int n = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) n += !isfinite(v[i]);
    dbg_count_nonfinite(n);
#else
    (void)v;
#endif
}
__device__ __forceinline__ void dbg_check4(float4 a) {
#ifdef W8A8_DEBUG
    dbg_count_nonfinite(!isfinite(a.x) + !isfinite(a.y) + !isfinite(a.z) + !isfinite(a.w));
#else
    (void)a;
#endif
}
// Non-finite values among 8 raw bf16 values (exponent bits all ones).
__device__ __forceinline__ void dbg_check_bf16x8(uint4 u) {
#ifdef W8A8_DEBUG
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    int n = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) n += ((w[i] & 0x7f80u) == 0x7f80u) + ((w[i] & 0x7f800000u) == 0x7f800000u);
    dbg_count_nonfinite(n);
#else
    (void)u;
#endif
}
__device__ __forceinline__ void dbg_check1(float a) {
#ifdef W8A8_DEBUG
    dbg_count_nonfinite(!isfinite(a));
#else
    (void)a;
#endif
}

}  // namespace w8a8
