// w8_sumsq.cuh -- the sum of squares of rms_norm, rounded once to fp32.
//
// The definition ("PyTorch integra Helion en vLLM para acelerar inferencia FP8", section
// "Patron de fusion del forward pass": rms_norm fused with the fp8 quant) is the exact
// sum of the squared bf16 values, rounded to fp32 (nearest, ties to even), so that the
// result does not depend on the order in which threads add.  Each square of a bf16 is
// exact in fp64; the squares are added as double-doubles (hi + lo, Knuth's TwoSum for
// every addition of a term or of a partial sum), which carries about 106 significant
// bits, and hi + lo is rounded once to fp32 by locating it between its two fp32
// neighbours.  The result is the correctly rounded fp32 of the exact sum unless that
// sum lies within about 2^-85 (relative) of an fp32 rounding midpoint without being on
// it -- which no sum of a few thousand bf16 squares of ordinary range does.
#pragma once
#include <cstdint>

namespace w8 {

struct DSum {
    double hi, lo;
};

// s + b with the rounding error of the leading addition kept in the trailing part
__device__ __forceinline__ DSum dsum_add(DSum s, double b)
{
    const double t = __dadd_rn(s.hi, b);
    const double bb = __dsub_rn(t, s.hi);
    const double err = __dadd_rn(__dsub_rn(s.hi, __dsub_rn(t, bb)), __dsub_rn(b, bb));
    return DSum{t, __dadd_rn(s.lo, err)};
}

__device__ __forceinline__ DSum dsum_add(DSum a, DSum b)
{
    DSum s = dsum_add(a, b.hi);
    s.lo = __dadd_rn(s.lo, b.lo);
    return s;
}

// one square of a bf16 value (exact in fp64) added to s
__device__ __forceinline__ DSum dsum_sq(DSum s, float x)
{
    const double d = (double)x;
    return dsum_add(s, __dmul_rn(d, d));
}

__device__ __forceinline__ DSum dsum_shfl_xor(DSum s, int o)
{
    return DSum{__shfl_xor_sync(0xFFFFFFFFu, s.hi, o), __shfl_xor_sync(0xFFFFFFFFu, s.lo, o)};
}

// hi + lo rounded once to fp32, to nearest, ties to even
__device__ __forceinline__ float dsum_to_f32(DSum a)
{
    // renormalise: v = RN(hi + lo), e = the exact remainder (|e| <= half an fp64 ulp of v)
    const double v = __dadd_rn(a.hi, a.lo);
    const double bb = __dsub_rn(v, a.hi);
    const double e = __dadd_rn(__dsub_rn(a.hi, __dsub_rn(v, bb)), __dsub_rn(a.lo, bb));
    const float dn = __double2float_rd(v), up = __double2float_ru(v);
    if (!(dn != up)) return dn;   // v is an fp32 value (or NaN): e cannot move it
    const double up_d = isinf(up) ? 0x1p128 : (double)up;
    // the midpoint of two neighbouring fp32 values is exact in fp64
    const double mid = __dmul_rn(0.5, __dadd_rn((double)dn, up_d));
    if (v < mid) return dn;
    if (v > mid) return up;
    if (e > 0.0) return up;
    if (e < 0.0) return dn;
    return (__float_as_uint(dn) & 1u) ? up : dn;
}

}  // namespace w8
