// dd.cuh -- double-double accumulation for the SSZ searches: error-free
// transformations (Knuth's TwoSum; the FMA TwoProduct where products are
// formed) so that sums of exact fp64 products keep ~106 bits.
#pragma once

#include "common.cuh"

namespace w8a8 {

struct dd {
    double hi, lo;
};

__device__ __forceinline__ dd two_sum(double a, double b) {
    const double s = a + b;
    const double bb = s - a;
    return {s, (a - (s - bb)) + (b - bb)};
}

// a += b (b a double-double), cascaded: exact in hi/lo pairs up to the
// rounding of the small lo sum.  TwoSum's error term is exact and symmetric
// in its arguments, so butterfly reductions give identical results on all
// lanes.
__device__ __forceinline__ dd dd_add_cascade(dd a, dd b) {
    const dd s = two_sum(a.hi, b.hi);
    return {s.hi, (a.lo + b.lo) + s.lo};
}

__device__ __forceinline__ void dd_acc(dd &a, double t) {
    const dd s = two_sum(a.hi, t);
    a.hi = s.hi;
    a.lo += s.lo;
}

__device__ __forceinline__ dd warp_sum_dd(dd a) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        a = dd_add_cascade(a, {__shfl_xor_sync(0xffffffffu, a.hi, o), __shfl_xor_sync(0xffffffffu, a.lo, o)});
    return a;
}

// Plain fp64 butterfly sum: every lane ends with the same value (a + b ==
// b + a exactly).
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// a * b as a double-double (exact: TwoProduct with one FMA).
__device__ __forceinline__ dd two_prod(double a, double b) {
    const double p = a * b;
    return {p, fma(a, b, -p)};
}

// x * (a double-double) with x exact in fp64; error ~2^-104 relative.
__device__ __forceinline__ dd dd_mul_d(dd a, double x) {
    const dd p = two_prod(a.hi, x);
    return {p.hi, p.lo + a.lo * x};
}

// Full double-double sum (renormalised).
__device__ __forceinline__ dd dd_add(dd a, dd b) {
    const dd s = two_sum(a.hi, b.hi);
    const double lo = s.lo + (a.lo + b.lo);
    return two_sum(s.hi, lo);
}

}  // namespace w8a8
