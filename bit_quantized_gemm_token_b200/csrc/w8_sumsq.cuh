// w8_sumsq.cuh -- the sum of squares of rms_norm, rounded once to fp32.
//
// The definition ("PyTorch integra Helion en vLLM para acelerar inferencia FP8", section
// "Patron de fusion del forward pass": rms_norm fused with the fp8 quant) is the exact
// sum of the squared bf16 values, rounded to fp32 (nearest, ties to even), so that the
// result does not depend on the order in which threads add.  Each square of a bf16 is
// exact in fp64.  A plain fp64 sum in any order, with its error bound, almost always
// settles the fp32 rounding (sq_round_certain below).  Otherwise the squares are added
// as double-doubles (hi + lo, Knuth's TwoSum for every
// addition of a term or of a partial sum), which carries about 106 significant bits, and
// hi + lo is rounded once to fp32 by locating it between its two fp32 neighbours: the
// correctly rounded fp32 of the exact sum unless that sum lies within about 2^-85
// (relative) of an fp32 rounding midpoint without being on it.
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

// Rounding certificate of a plain fp64 sum of squares.  The fp64 sum s of nonnegative
// terms (each square of a bf16 is exact in fp64) added in any order in which no term
// passes through more than d roundings differs from the exact sum S by at most
// gamma_d S, gamma_d = d u / (1 - d u), u = 2^-53 (the standard bound for recursive and
// pairwise summation; any order of n terms has d <= n - 1).  With d u <= 1/4 that puts S
// in [s - e, s + e], e = d 2^-52 s.  RN to fp32 is monotone, so when both ends of the
// interval (rounded outward in fp64) round to the same fp32, S rounds to it as well:
// that value is the correctly rounded exact sum, whatever the order of the fp64
// additions.  A non-finite s is already the answer: squares of finite bf16 values (below
// 2^256) cannot overflow an fp64 sum, so s = +inf means an infinite input (the exact sum
// is +inf) and NaN a NaN input.  The test fails only for an S within about d 2^-52
// (relative) of an fp32 rounding midpoint; the caller then recomputes with double-doubles.
__device__ __forceinline__ bool sq_round_certain(double s, int depth, float* out)
{
    const double e = __dmul_ru(s, (double)depth * 0x1p-52);
    const float lo = __double2float_rn(__dsub_rd(s, e));
    const float hi = __double2float_rn(__dadd_ru(s, e));
    if (!isfinite(s)) {
        *out = __double2float_rn(s);
        return true;
    }
    *out = lo;
    return lo == hi;
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
