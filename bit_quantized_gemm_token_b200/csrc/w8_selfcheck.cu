// w8_selfcheck.cu -- a device-side check of the division-free quotient that every
// quantizer uses (w8_codes.cuh, quotient_rn) against the IEEE division __fdiv_rn.
//
// The codes are defined from the correctly rounded quotient x / s; the kernels multiply
// by a prepared reciprocal and correct the result with one fused multiply-add
// (Markstein's method; the shorter plain form where no scaling is needed and the row's
// maximum is finite, one value at a time and paired on the f32x2 instructions).  The two must give the same 8-bit code for every input a
// quantizer can meet, and the same fp32 quotient wherever a code can depend on it
// (|x / s| >= 2^-10).
//   modes 0, 1, 2 (bf16 numerators: the plain quantizers): every bf16 amax from the
//     smallest subnormal to +inf, every bf16 x with |x| <= amax, both signs -- about
//     1.1e9 pairs per scale rule (amax / 448 for e4m3, amax / 127 for int8, UE8M0);
//   modes 3, 4, 5 (fp32 numerators: rms_norm and silu_and_mul outputs), same rules:
//     2^30 pairs from a counter-based hash -- a random finite amax, then x either a
//     random fp32 of magnitude <= amax or one within 3 ulps of (a code's rounding
//     midpoint) * s, the inputs where a wrong last bit of the quotient flips a code.
#include "w8_codes.cuh"
#include "w8_internal.h"

namespace w8 {
namespace {

struct CheckOut {
    unsigned long long* bad;
    unsigned int* first;   // [0] amax bits, [1] x bits of one failing pair
};

__device__ __forceinline__ void compare(int rule, float amax, float s, const RowDivisor& d, float x,
                                        unsigned long long& bad, uint32_t& fa, uint32_t& fx, uint32_t abits,
                                        uint32_t xbits)
{
    const float q1 = __fdiv_rn(x, s);
    const float q2 = quotient_rn(x, d);
    // the plain form wherever the quantizers take it (no scaling, finite amax), scalar and
    // paired (with -x beside x)
    float q3 = q2;
    bool pair_bad = false;   // the paired form differs from the scalar one in any bit
    if (d.plain) {
        q3 = quotient_plain(x, d);
        float p0, p1;
        quotient_plain2(x, -x, d, p0, p1);
        pair_bad = __float_as_uint(p0) != __float_as_uint(q3) ||
                   __float_as_uint(p1) != __float_as_uint(quotient_plain(-x, d));
    }
    const uint32_t c1 = rule == 1 ? int8_code(q1) : (e4m3x2(q1, 0.0f) & 0xFFu);
    const uint32_t c2 = rule == 1 ? int8_code(q2) : (e4m3x2(q2, 0.0f) & 0xFFu);
    const uint32_t c3 = rule == 1 ? int8_code(q3) : (e4m3x2(q3, 0.0f) & 0xFFu);
    // the quotient must match wherever a code can depend on it: |x / s| >= 2^-10
    const bool coded = fabsf(q1) >= 0x1p-10f && isfinite(q1);
    if (pair_bad || c1 != c2 || c1 != c3 ||
        (coded && (__float_as_uint(q1) != __float_as_uint(q2) || __float_as_uint(q1) != __float_as_uint(q3)))) {
        ++bad;
        fa = abits;
        fx = xbits;
    }
    (void)amax;
}

__device__ __forceinline__ void flush(const CheckOut& o, unsigned long long bad, uint32_t fa, uint32_t fx)
{
    if (bad) {
        atomicAdd(o.bad, bad);
        if (atomicCAS(o.first, 0u, fa | 0x80000000u) == 0u) o.first[1] = fx;
    }
}

__global__ void __launch_bounds__(256) quotient_check_bf16(int rule, CheckOut o)
{
    // block b: amax = the positive bf16 with bit pattern b + 1 (0x0001 .. 0x7F80 = +inf)
    const uint32_t ab = blockIdx.x + 1;
    const float amax = __uint_as_float(ab << 16);
    const float s = scale_from_amax(amax, rule == 1 ? kInt8Max : kE4M3Max, rule == 2);
    const RowDivisor d = make_divisor(s, amax);
    unsigned long long bad = 0;
    uint32_t fa = 0, fx = 0;
    // positive bf16 values order like their bit patterns: x runs over 0 .. amax
    for (uint32_t xb = threadIdx.x; xb <= ab; xb += blockDim.x) {
#pragma unroll
        for (uint32_t sign = 0; sign <= 0x8000u; sign += 0x8000u) {
            const uint32_t bits = (xb | sign) << 16;
            compare(rule, amax, s, d, __uint_as_float(bits), bad, fa, fx, ab << 16, bits);
        }
    }
    flush(o, bad, fa, fx);
}

// a 32-bit mixing function (the finaliser of MurmurHash3) over a running counter
__device__ __forceinline__ uint32_t mix32(uint32_t h)
{
    h ^= h >> 16;
    h *= 0x85EBCA6Bu;
    h ^= h >> 13;
    h *= 0xC2B2AE35u;
    h ^= h >> 16;
    return h;
}

// value of the positive e4m3 code b (0 .. 0x7E)
__device__ __forceinline__ float e4m3_value(uint32_t b)
{
    const uint32_t E = b >> 3, M = b & 7u;
    return E == 0 ? ldexpf((float)M, -9) : ldexpf((float)(8u + M), (int)E - 10);
}

constexpr int kFp32Iters = 256;

__global__ void __launch_bounds__(256) quotient_check_fp32(int rule, CheckOut o)
{
    unsigned long long bad = 0;
    uint32_t fa = 0, fx = 0;
    uint32_t ctr = ((blockIdx.x * 256u + threadIdx.x) * kFp32Iters) * 4u + (uint32_t)rule * 0x9E3779B9u;
    for (int it = 0; it < kFp32Iters; ++it) {
        const uint32_t h0 = mix32(ctr++), h1 = mix32(ctr++), h2 = mix32(ctr++), h3 = mix32(ctr++);
        const uint32_t abits = 1u + h0 % 0x7F7FFFFFu;   // a positive finite amax
        const float amax = __uint_as_float(abits);
        const float s = scale_from_amax(amax, rule == 1 ? kInt8Max : kE4M3Max, rule == 2);
        const RowDivisor d = make_divisor(s, amax);
        uint32_t xbits;
        if (h1 & 1u) {
            xbits = h2 % (abits + 1u);   // |x| <= amax, uniform over bit patterns
        } else {
            // near the midpoint between two neighbouring codes, times s
            float mid;
            if (rule == 1) {
                mid = (float)(h2 % 127u) + 0.5f;
            } else {
                const uint32_t b = h2 % 0x7Eu;
                mid = 0.5f * (e4m3_value(b) + e4m3_value(b + 1u));
            }
            const int delta = (int)(h3 % 7u) - 3;
            xbits = (uint32_t)max(0, (int)__float_as_uint(__fmul_rn(mid, s)) + delta);
            if (xbits > abits) xbits = abits;
        }
        xbits |= (h1 & 2u) << 30;   // sign
        compare(rule, amax, s, d, __uint_as_float(xbits), bad, fa, fx, abits, xbits);
    }
    flush(o, bad, fa, fx);
}

}  // namespace
}  // namespace w8

using namespace w8;

extern "C" int w8_selfcheck_quotient(int mode, unsigned long long* mismatches, unsigned int* first_bad,
                                     w8_stream_t stream)
{
    if (mode < 0 || mode > 5 || !mismatches || !first_bad) return W8_ERR_INVALID_ARG;
    int rc = check_device(nullptr);
    if (rc != W8_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const CheckOut o{mismatches, first_bad};
    if (mode < 3)
        quotient_check_bf16<<<0x7F80, 256, 0, s>>>(mode, o);
    else
        quotient_check_fp32<<<(1u << 30) / (256u * kFp32Iters), 256, 0, s>>>(mode - 3, o);
    return cudaGetLastError() == cudaSuccess ? W8_OK : W8_ERR_CUDA;
}
