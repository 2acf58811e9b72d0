// w8_codes.cuh -- scalar pieces of the 8-bit quantizers shared by the quantizer kernels
// and the GEMM's fused activation quantization: bf16 unpacking, the e4m3 / int8 encoders,
// the scale rule and a correctly rounded quotient x / s.
//
// Scales and codes ("PyTorch integra Helion en vLLM para acelerar inferencia FP8",
// section "Kernels Helion implementados"; "Helion DSL added to vLLM to autotune linear
// inference backends", section "Unified GEMM Architecture"): s = amax / 448 (e4m3) or
// amax / 127 (int8), an IEEE fp32 division; s = 1 for an all-zero row or group; UE8M0
// scales are the smallest power of two not below amax / 448; codes = RNE(x / s),
// saturating, with x / s rounded once to fp32.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cstdint>

#include "w8.h"

namespace w8 {

constexpr float kE4M3Max = 448.0f;
constexpr float kInt8Max = 127.0f;

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float (&f)[8])
{
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xFFFF0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xFFFF0000u);
    f[4] = __uint_as_float(v.z << 16);
    f[5] = __uint_as_float(v.z & 0xFFFF0000u);
    f[6] = __uint_as_float(v.w << 16);
    f[7] = __uint_as_float(v.w & 0xFFFF0000u);
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p)
{
    return __ldg(reinterpret_cast<const uint4*>(p));
}

// Two fp32 -> two e4m3 codes (round to nearest even, saturating); element `lo` in the
// low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi)
{
    return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ uint32_t int8_code(float v)
{
    int r = __float2int_rn(v);   // ties to even; NaN -> 0
    r = max(-127, min(127, r));
    return static_cast<uint32_t>(r) & 0xFFu;
}

// Correctly rounded x / s for the quantizers, without a division per element.  The row's
// divisor is prepared once: y = RN(1 / s') with s' = s, or s * 2^64 when s is below 2^-92
// (x is scaled by the same exact power of two).  Per element (Markstein's theorem,
// P. Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990; J.-M. Muller et al., "Handbook of
// Floating-Point Arithmetic", ch. on division with an FMA):
//   q0 = RN(x * y);  r = x - q0 * s' (one fma);  q = RN(q0 + r * y)
// is the correctly rounded quotient whenever the remainder r is exact.  r is a multiple
// of ulp(q0) ulp(s'), so it is an fp32 value when that product is at least 2^-149: with
// s' >= 2^-92 this holds for every |q0| >= 2^-10, and smaller quotients give a zero code
// in both formats (e4m3 rounds values up to 2^-10 to zero, int8 values below 1/2).  So
// the codes, and the quotient wherever a code can depend on it, are those of IEEE
// division; the sign of x is copied onto q so that -0 stays -0.  Checked on the device
// against __fdiv_rn (w8_selfcheck.cu): every bf16 x with every bf16 amax, infinities
// included, |x| <= amax (amax / 448, amax / 127, UE8M0), and 2^30 fp32 numerators per
// scale rule, half of them within a few ulps of a code's rounding boundary.
struct RowDivisor {
    float s;      // s' (s, or s * 2^64)
    float y;      // RN(1 / s')
    float f;      // 1, or 2^64: the factor applied to x
    bool plain;   // f = 1 and no element of the row is infinite: quotient_plain applies
};

__device__ __forceinline__ RowDivisor make_divisor(float s)
{
    RowDivisor d;
    const bool tiny = s < 0x1p-92f;
    d.f = tiny ? 0x1p64f : 1.0f;
    d.s = __fmul_rn(s, d.f);
    d.y = __frcp_rn(d.s);
    // s = +inf (an infinite amax): y = 0, and s' = 0 keeps the correction finite, so a
    // finite x gives +-0 and an infinite x NaN, as x / inf does
    if (isinf(s)) d.s = 0.0f;
    d.plain = false;
    return d;
}

// The same divisor for a row (or group) whose maximum magnitude amax is known: when no
// scaling is needed and amax is finite (so no element is infinite and q0 never is),
// quotient_plain gives quotient_rn's result with two operations fewer per element.
__device__ __forceinline__ RowDivisor make_divisor(float s, float amax)
{
    RowDivisor d = make_divisor(s);
    d.plain = d.f == 1.0f && isfinite(amax) && !isinf(s);
    return d;
}

__device__ __forceinline__ float quotient_rn(float x, const RowDivisor& d)
{
    const float xs = __fmul_rn(x, d.f);
    const float q0 = __fmul_rn(xs, d.y);
    const float r = __fmaf_rn(-q0, d.s, xs);
    // an infinite q0 comes only from an infinite x over a finite s: the quotient is q0
    return copysignf(fabsf(q0) == INFINITY ? q0 : __fmaf_rn(r, d.y, q0), x);
}

// quotient_rn for a divisor with d.plain set (x finite or NaN, no scaling)
__device__ __forceinline__ float quotient_plain(float x, const RowDivisor& d)
{
    const float q0 = __fmul_rn(x, d.y);
    const float r = __fmaf_rn(-q0, d.s, x);
    return copysignf(__fmaf_rn(r, d.y, q0), x);
}

// 8 values / s -> 8 codes packed little-endian into a uint2 (d = make_divisor(s)).
// quotient_plain of two values at once on the paired fp32 instructions of sm_100
// (fma.rn.f32x2 / mul.rn.f32x2: each half the same correctly rounded operation, so each
// quotient equals quotient_plain's)
__device__ __forceinline__ void quotient_plain2(float x0, float x1, const RowDivisor& d, float& q0, float& q1)
{
    const unsigned long long X = ((unsigned long long)__float_as_uint(x1) << 32) | __float_as_uint(x0);
    const unsigned long long Y = ((unsigned long long)__float_as_uint(d.y) << 32) | __float_as_uint(d.y);
    const unsigned long long NS = ((unsigned long long)__float_as_uint(-d.s) << 32) | __float_as_uint(-d.s);
    unsigned long long Q, R, Z;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(Q) : "l"(X), "l"(Y));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(R) : "l"(Q), "l"(NS), "l"(X));   // x - q0 s', exact
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(Z) : "l"(R), "l"(Y), "l"(Q));
    q0 = copysignf(__uint_as_float((uint32_t)Z), x0);
    q1 = copysignf(__uint_as_float((uint32_t)(Z >> 32)), x1);
}

template <int QFMT>
__device__ __forceinline__ uint2 encode8(const float (&f)[8], const RowDivisor& d)
{
    float v[8];
    if (d.plain) {
#pragma unroll
        for (int i = 0; i < 8; i += 2) quotient_plain2(f[i], f[i + 1], d, v[i], v[i + 1]);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = quotient_rn(f[i], d);
    }
    uint2 r;
    if (QFMT == W8_Q_FP8) {
        r.x = e4m3x2(v[0], v[1]) | (e4m3x2(v[2], v[3]) << 16);
        r.y = e4m3x2(v[4], v[5]) | (e4m3x2(v[6], v[7]) << 16);
    } else {
        r.x = int8_code(v[0]) | (int8_code(v[1]) << 8) | (int8_code(v[2]) << 16) | (int8_code(v[3]) << 24);
        r.y = int8_code(v[4]) | (int8_code(v[5]) << 8) | (int8_code(v[6]) << 16) | (int8_code(v[7]) << 24);
    }
    return r;
}

__device__ __forceinline__ float scale_from_amax(float amax, float qmax, bool ue8m0)
{
    if (!(amax > 0.0f)) return 1.0f;
    float r = __fdiv_rn(amax, qmax);
    if (!ue8m0) return r;
    int e;
    float f = frexpf(r, &e);          // r = f * 2^e exactly, f in [0.5, 1)
    int p = (f == 0.5f) ? e - 1 : e;  // smallest power of two >= r
    p = max(-127, min(127, p));
    return ldexpf(1.0f, p);
}

}  // namespace w8
