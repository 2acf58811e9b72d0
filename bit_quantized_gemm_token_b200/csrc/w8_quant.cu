// w8_quant.cu -- activation quantizers and the fused rms_norm / silu_and_mul producers.
//
// Definitions (the pages name these kernels in "PyTorch integra Helion en vLLM para
// acelerar inferencia FP8", section "Kernels Helion implementados": dynamic_per_token_
// scaled_fp8_quant, per_token_group_fp8_quant, rms_norm_dynamic_per_token_quant,
// silu_and_mul_dynamic_per_token_quant; the fusions are the two pairs of section
// "Patron de fusion del forward pass"):
//   s = amax / Q (fp32 division; Q = 448 e4m3, 127 int8; s = 1 for an all-zero row),
//   q = e4m3_rn_satfinite(x / s)  or  clamp(rint(x / s), -127, 127),
//   UE8M0 scales: the smallest power of two >= amax/448, exponent in [-127, 127].
// Every quotient x / s is the correctly rounded IEEE one: silu's division is __fdiv_rn,
// and the codes take x / s from a row reciprocal with Markstein's correction
// (w8_codes.cuh, quotient_rn: the same fp32 quotient wherever a code can depend on it).
// No arithmetic is left to compiler contraction (__fmul_rn / __fadd_rn / __fmaf_rn spell
// out each rounding), so the codes are a deterministic function of the inputs.
//
// Layout of the work: the row kernels give one CTA per row and keep the row in
// registers (16-byte vector loads, CPT chunks of 8 bf16 per thread); reductions are
// warp shuffles plus one shared-memory stage.  The group kernel gives a half-warp per
// 128-element group.  Under programmatic dependent launch every kernel releases its
// dependents at entry (so the next GEMM can start streaming its weights) and waits for
// the previous grid before it reads or writes anything.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <map>
#include <mutex>

#include "w8_codes.cuh"
#include "w8_internal.h"
#include "w8_ptx.cuh"
#include "w8_sumsq.cuh"

namespace w8 {
namespace {

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Max over the CTA; every thread receives the result.  `red` holds 32 floats.
__device__ __forceinline__ float block_max(float v, float* red)
{
    v = warp_max(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) red[w] = v;
    __syncthreads();
    float r = (l < (int)(blockDim.x >> 5)) ? red[l] : 0.0f;
    r = warp_max(r);
    __syncthreads();
    return r;
}

// fp64 sum over the CTA (a fixed tree); every thread gets the result.  `red` holds 32.
__device__ __forceinline__ double block_sum64(double v, double* red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) red[w] = v;
    __syncthreads();
    double r = (l < (int)(blockDim.x >> 5)) ? red[l] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) r = __dadd_rn(r, __shfl_xor_sync(0xFFFFFFFFu, r, o));
    __syncthreads();
    return r;
}

// Double-double sum over the CTA; every thread gets the result.  `red` holds 32 DSums.
__device__ __forceinline__ DSum block_sum_dd(DSum v, DSum* red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = dsum_add(v, dsum_shfl_xor(v, o));
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) red[w] = v;
    __syncthreads();
    DSum r = (l < (int)(blockDim.x >> 5)) ? red[l] : DSum{0.0, 0.0};
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) r = dsum_add(r, dsum_shfl_xor(r, o));
    __syncthreads();
    return r;
}

// exp(x) in fp32 by Cody & Waite's method: x = n ln2 + r with n = rint(x log2 e) and
// ln2 split into a short leading part and a remainder, exp(r) by its Taylor series to
// degree 7 (Horner, fused multiply-adds), and the exact scaling by 2^n as two
// power-of-two factors that stay normal.  Each step is an explicitly rounded fp32 op,
// so the result is fully specified (worst error about 1 ulp against exp).  It is computed
// for two values at once (exp_cw2 below).

// Two fp32 values in one 64-bit register, for the paired fp32 instructions of sm_100
// (fma.rn.f32x2 / mul.rn.f32x2: each half an independent, correctly rounded operation)
__device__ __forceinline__ unsigned long long f2pack(float a, float b)
{
    return ((unsigned long long)__float_as_uint(b) << 32) | __float_as_uint(a);
}
__device__ __forceinline__ float f2lo(unsigned long long v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float f2hi(unsigned long long v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b, unsigned long long c)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// The exp described above, for two values at once: each gets the same sequence of
// correctly rounded operations, paired (half the instructions for the reduction, the
// polynomial and the scaling; 115 -> 109 us for silu_and_mul + quant at 4096 x 12288 on
// B200).  NaN gives
// NaN, x > 100 gives +inf and x < -150 gives 0; those inputs run the normal path on a
// clamped value first.
__device__ __forceinline__ void exp_cw2(float x0, float x1, float& e0, float& e1)
{
    const float c0 = fminf(fmaxf(x0, -150.0f), 100.0f), c1 = fminf(fmaxf(x1, -150.0f), 100.0f);
    const unsigned long long X = f2pack(c0, c1);
    const unsigned long long T = mul2(X, f2pack(0x1.715476p+0f, 0x1.715476p+0f));   // log2(e)
    const float n0 = rintf(f2lo(T)), n1 = rintf(f2hi(T));
    const unsigned long long NN = f2pack(-n0, -n1);
    unsigned long long R = fma2(NN, f2pack(0x1.62e400p-1f, 0x1.62e400p-1f), X);     // ln 2, leading bits
    R = fma2(NN, f2pack(0x1.7f7d1cp-20f, 0x1.7f7d1cp-20f), R);                      // ln 2, remainder
    unsigned long long P = f2pack(0x1.a01a02p-13f, 0x1.a01a02p-13f);                // 1/7!
    P = fma2(P, R, f2pack(0x1.6c16c2p-10f, 0x1.6c16c2p-10f));
    P = fma2(P, R, f2pack(0x1.111112p-7f, 0x1.111112p-7f));
    P = fma2(P, R, f2pack(0x1.555556p-5f, 0x1.555556p-5f));
    P = fma2(P, R, f2pack(0x1.555556p-3f, 0x1.555556p-3f));
    P = fma2(P, R, f2pack(0.5f, 0.5f));
    P = fma2(P, R, f2pack(1.0f, 1.0f));
    P = fma2(P, R, f2pack(1.0f, 1.0f));
    const int i0 = (int)n0, i1 = (int)n1;
    const int a0 = i0 / 2, a1 = i1 / 2;
    P = mul2(P, f2pack(__int_as_float((a0 + 127) << 23), __int_as_float((a1 + 127) << 23)));
    P = mul2(P, f2pack(__int_as_float((i0 - a0 + 127) << 23), __int_as_float((i1 - a1 + 127) << 23)));
    e0 = f2lo(P);
    e1 = f2hi(P);
    if (x0 != x0) e0 = x0; else if (x0 > 100.0f) e0 = __int_as_float(0x7F800000); else if (x0 < -150.0f) e0 = 0.0f;
    if (x1 != x1) e1 = x1; else if (x1 > 100.0f) e1 = __int_as_float(0x7F800000); else if (x1 < -150.0f) e1 = 0.0f;
}

// Grouped (1x128) variant of the last step of the row kernels: the 16 chunks of a
// 128-element group sit in 16 consecutive lanes (chunk index = thread + c * blockDim,
// blockDim a multiple of 32), so the group's amax is a half-warp reduction.  Writes the
// chunk's 8 codes and, from the group's first lane, its scale.
__device__ __forceinline__ void encode_chunk_grouped(const float (&y)[8], int idx, int ng, bool ue8m0,
                                                     uint8_t* qrow, float* srow)
{
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(y[i]));
    const unsigned hmask = 0xFFFFu << (threadIdx.x & 16);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(hmask, amax, o));
    const float s = scale_from_amax(amax, kE4M3Max, ue8m0);
    if ((idx & 15) == 0) srow[idx >> 4] = s;
    (void)ng;
    const RowDivisor d = make_divisor(s, amax);
    *reinterpret_cast<uint2*>(qrow + (size_t)idx * 8) = encode8<W8_Q_FP8>(y, d);
}

// ------------------------------------------------------------------- per-token rows
// Rows m = blockIdx.x, + gridDim.x, ...: each CTA issues the loads of its next row before
// it reduces and encodes the current one, so its loads stay in flight across the row's
// barriers (the grid is one row per CTA for few rows, the resident CTAs for many).
template <int CPT>
__device__ __forceinline__ void load_row(const __nv_bfloat16* xr, int chunks, uint4 (&r)[CPT])
{
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        const int idx = threadIdx.x + c * blockDim.x;
        if (idx < chunks) r[c] = ld_nc_v4(xr + (size_t)idx * 8);
    }
}

template <int QFMT, int CPT>
__global__ void __launch_bounds__(1024) quant_rows_kernel(const __nv_bfloat16* __restrict__ x, int M, int K, int ldx,
                                                          uint8_t* __restrict__ q, float* __restrict__ scale)
{
    __shared__ float red[32];
    ptx::grid_dep_launch();   // dependents may launch now; they wait for this grid themselves
    ptx::grid_dep_wait();
    const int chunks = K >> 3;
    uint4 raw[CPT], nxt[CPT];
    int m = blockIdx.x;
    load_row<CPT>(x + (size_t)m * ldx, chunks, raw);
    for (;;) {
        const int mn = m + (int)gridDim.x;
        if (mn < M) load_row<CPT>(x + (size_t)mn * ldx, chunks, nxt);
        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            const int idx = threadIdx.x + c * blockDim.x;
            if (idx < chunks) {
                float f[8];
                unpack_bf16x8(raw[c], f);
#pragma unroll
                for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
            }
        }
        amax = block_max(amax, red);
        const float s = scale_from_amax(amax, QFMT == W8_Q_FP8 ? kE4M3Max : kInt8Max, false);
        if (threadIdx.x == 0) scale[m] = s;
        const RowDivisor d = make_divisor(s, amax);
        uint8_t* qr = q + (size_t)m * K;
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            const int idx = threadIdx.x + c * blockDim.x;
            if (idx < chunks) {
                float f[8];
                unpack_bf16x8(raw[c], f);
                *reinterpret_cast<uint2*>(qr + (size_t)idx * 8) = encode8<QFMT>(f, d);
            }
        }
        if (mn >= M) break;
        m = mn;
#pragma unroll
        for (int c = 0; c < CPT; ++c) raw[c] = nxt[c];
    }
}

// ------------------------------------------------------------------- 1x128 groups
// A half-warp (16 lanes x 8 elements) per group; scale[m * (K/128) + g].  (Four groups
// per half-warp with their loads issued together measured slower on B200: 70 against
// 64 us for 16384 x 4096.)
__global__ void __launch_bounds__(256) quant_group128_kernel(const __nv_bfloat16* __restrict__ x, int M, int K,
                                                             int ldx, uint8_t* __restrict__ q,
                                                             float* __restrict__ scale, int ue8m0)
{
    ptx::grid_dep_launch();   // dependents may launch now; they wait for this grid themselves
    ptx::grid_dep_wait();
    const int gpr = K >> 7;
    const long long total = (long long)M * gpr;
    const long long gid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
    const int l16 = threadIdx.x & 15;
    const unsigned hmask = 0xFFFFu << (threadIdx.x & 16);
    if (gid >= total) return;   // whole half-warps leave together
    const int m = (int)(gid / gpr), g = (int)(gid % gpr);
    const uint4 raw = ld_nc_v4(x + (size_t)m * ldx + (size_t)g * 128 + l16 * 8);
    float f[8];
    unpack_bf16x8(raw, f);
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(hmask, amax, o));
    const float s = scale_from_amax(amax, kE4M3Max, ue8m0 != 0);
    if (l16 == 0) scale[(size_t)m * gpr + g] = s;
    const RowDivisor d = make_divisor(s, amax);
    *reinterpret_cast<uint2*>(q + (size_t)m * K + (size_t)g * 128 + l16 * 8) = encode8<W8_Q_FP8>(f, d);
}

// ------------------------------------------------------------------- 128x128 weight blocks
__global__ void __launch_bounds__(256) quant_weight_block_kernel(const __nv_bfloat16* __restrict__ w, int N, int K,
                                                                 uint8_t* __restrict__ q, float* __restrict__ scale,
                                                                 int ue8m0)
{
    __shared__ float red[32];
    ptx::grid_dep_launch();   // dependents may launch now; they wait for this grid themselves
    ptx::grid_dep_wait();
    const int bk = blockIdx.x, bn = blockIdx.y;
    const int nbk = gridDim.x;
    const int rows = min(128, N - bn * 128), cols = min(128, K - bk * 128);
    uint4 raw[8];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int c = threadIdx.x + i * 256;   // 16 chunks of 8 per row
        const int r = c >> 4, cc = (c & 15) * 8;
        if (r < rows && cc < cols) {
            raw[i] = ld_nc_v4(w + (size_t)(bn * 128 + r) * K + bk * 128 + cc);
            float f[8];
            unpack_bf16x8(raw[i], f);
#pragma unroll
            for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
        }
    }
    amax = block_max(amax, red);
    const float s = scale_from_amax(amax, kE4M3Max, ue8m0 != 0);
    if (threadIdx.x == 0) scale[(size_t)bn * nbk + bk] = s;
    const RowDivisor d = make_divisor(s, amax);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int c = threadIdx.x + i * 256;
        const int r = c >> 4, cc = (c & 15) * 8;
        if (r < rows && cc < cols) {
            float f[8];
            unpack_bf16x8(raw[i], f);
            *reinterpret_cast<uint2*>(q + (size_t)(bn * 128 + r) * K + bk * 128 + cc) = encode8<W8_Q_FP8>(f, d);
        }
    }
}

// ------------------------------------------------------------------- rms_norm + quant
template <int CPT, bool GROUPED>
__global__ void __launch_bounds__(1024) rmsnorm_quant_kernel(const __nv_bfloat16* __restrict__ x,
                                                             const __nv_bfloat16* __restrict__ gamma, float eps,
                                                             int M, int H, int ldx, uint8_t* __restrict__ q,
                                                             float* __restrict__ scale, int ue8m0)
{
    __shared__ DSum redd[32];
    __shared__ double red64[32];
    __shared__ float red[32];
    ptx::grid_dep_launch();   // dependents may launch now; they wait for this grid themselves
    ptx::grid_dep_wait();
    (void)M;
    const int m = blockIdx.x;
    const int chunks = H >> 3;
    uint4 raw[CPT];
    load_row<CPT>(x + (size_t)m * ldx, chunks, raw);
    double ss64 = 0.0;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        const int idx = threadIdx.x + c * blockDim.x;
        if (idx < chunks) {
            float f[8];
            unpack_bf16x8(raw[c], f);
#pragma unroll
            for (int i = 0; i < 8; ++i) ss64 = __fma_rn((double)f[i], (double)f[i], ss64);   // squares exact
        }
    }
    // the exact sum of squares rounded once to fp32 (w8_sumsq.cuh): the fp64 sum when its
    // error bound settles the rounding (no term meets more than H roundings), else the
    // double-double sum; the CTA-wide sum is the same in every thread, so is the branch
    ss64 = block_sum64(ss64, red64);
    float ssf;
    if (!sq_round_certain(ss64, H, &ssf)) {
        DSum ss{0.0, 0.0};
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            const int idx = threadIdx.x + c * blockDim.x;
            if (idx < chunks) {
                float f[8];
                unpack_bf16x8(raw[c], f);
#pragma unroll
                for (int i = 0; i < 8; ++i) ss = dsum_sq(ss, f[i]);
            }
        }
        ssf = dsum_to_f32(block_sum_dd(ss, redd));
    }
    const float mean = __fdiv_rn(ssf, (float)H);
    const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(mean, eps)));
    // y = (x * r) * gamma, kept in registers for the codes
    float y[CPT][8];
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        const int idx = threadIdx.x + c * blockDim.x;
        if (idx < chunks) {
            float f[8], g[8];
            unpack_bf16x8(raw[c], f);
            unpack_bf16x8(ld_nc_v4(gamma + (size_t)idx * 8), g);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                y[c][i] = __fmul_rn(__fmul_rn(f[i], r), g[i]);
                amax = fmaxf(amax, fabsf(y[c][i]));
            }
        }
    }
    if (GROUPED) {
        // rms_norm_per_block_quant: one scale per 1x128 group of y
        const int ng = H >> 7;
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            const int idx = threadIdx.x + c * blockDim.x;
            if (idx < chunks) encode_chunk_grouped(y[c], idx, ng, ue8m0 != 0, q + (size_t)m * H, scale + (size_t)m * ng);
        }
        return;
    }
    amax = block_max(amax, red);
    const float s = scale_from_amax(amax, kE4M3Max, false);
    if (threadIdx.x == 0) scale[m] = s;
    const RowDivisor d = make_divisor(s, amax);
    uint8_t* qr = q + (size_t)m * H;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        const int idx = threadIdx.x + c * blockDim.x;
        if (idx < chunks) *reinterpret_cast<uint2*>(qr + (size_t)idx * 8) = encode8<W8_Q_FP8>(y[c], d);
    }
}

// ------------------------------------------------------------------- silu_and_mul + quant
template <int CPT, bool GROUPED>
__device__ __forceinline__ void silu_row(const uint4 (&rg)[CPT], const uint4 (&ru)[CPT], int m, int I, uint8_t* q,
                                         float* scale, int ue8m0, float* red)
{
    const int chunks = I >> 3;
    float h[CPT][8];
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        const int idx = threadIdx.x + c * blockDim.x;
        if (idx < chunks) {
            float g[8], u[8];
            unpack_bf16x8(rg[c], g);
            unpack_bf16x8(ru[c], u);
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                float e0, e1;
                exp_cw2(-g[i], -g[i + 1], e0, e1);
                h[c][i] = __fmul_rn(__fdiv_rn(g[i], __fadd_rn(1.0f, e0)), u[i]);
                h[c][i + 1] = __fmul_rn(__fdiv_rn(g[i + 1], __fadd_rn(1.0f, e1)), u[i + 1]);
                amax = fmaxf(amax, fmaxf(fabsf(h[c][i]), fabsf(h[c][i + 1])));
            }
        }
    }
    if (GROUPED) {
        // silu_and_mul_per_block_quant: one scale per 1x128 group of h
        const int ng = I >> 7;
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            const int idx = threadIdx.x + c * blockDim.x;
            if (idx < chunks) encode_chunk_grouped(h[c], idx, ng, ue8m0 != 0, q + (size_t)m * I, scale + (size_t)m * ng);
        }
        return;
    }
    amax = block_max(amax, red);
    const float s = scale_from_amax(amax, kE4M3Max, false);
    if (threadIdx.x == 0) scale[m] = s;
    const RowDivisor d = make_divisor(s, amax);
    uint8_t* qr = q + (size_t)m * I;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        const int idx = threadIdx.x + c * blockDim.x;
        if (idx < chunks) *reinterpret_cast<uint2*>(qr + (size_t)idx * 8) = encode8<W8_Q_FP8>(h[c], d);
    }
}

template <int CPT, bool GROUPED>
__global__ void __launch_bounds__(1024) silu_mul_quant_kernel(const __nv_bfloat16* __restrict__ xgu, int M, int I,
                                                              int ld, uint8_t* __restrict__ q,
                                                              float* __restrict__ scale, int ue8m0)
{
    __shared__ float red[32];
    ptx::grid_dep_launch();   // dependents may launch now; they wait for this grid themselves
    ptx::grid_dep_wait();
    (void)M;
    const int m = blockIdx.x;
    const int chunks = I >> 3;
    uint4 rg[CPT], ru[CPT];
    load_row<CPT>(xgu + (size_t)m * ld, chunks, rg);
    load_row<CPT>(xgu + (size_t)m * ld + I, chunks, ru);
    silu_row<CPT, GROUPED>(rg, ru, m, I, q, scale, ue8m0, red);
}

// Threads per row and chunks per thread for `rows` rows of `chunks` 16-byte chunks.  Each
// thread issues all its loads before the row's reductions.  Few rows (decode) are bound by
// the latency of one CTA's chain of loads, reductions and stores: the fewest chunks per
// thread (1, 2 or 4) that fits in 1024 threads keeps that chain short.  Many rows are
// bound by HBM: the most chunks per thread (4, 2 or 1) that still leaves 64 threads puts
// more bytes in flight per SM, whose thread slots run out before its CTA slots (16384
// rows of 4096 bf16: 63 -> 51 us on B200, while 32 rows lose ~4 us to the longer chain).
constexpr int kManyRows = 1024;

inline bool row_shape(int rows, int chunks, int* threads, int* cpt, int many_max = 4)
{
    static const int few[3] = {1, 2, 4}, many[3] = {4, 2, 1};
    const int* order = rows >= kManyRows ? many : few;
    for (int i = 0; i < 3; ++i) {
        const int c = order[i];
        const int t = (chunks + c - 1) / c;
        if (t > 1024) continue;
        if (rows >= kManyRows && ((t < 64 && c > 1) || (c > many_max && (chunks + many_max - 1) / many_max <= 1024)))
            continue;
        *cpt = c;
        *threads = ((t + 31) / 32) * 32;
        if (*threads < 64) *threads = 64;
        return true;
    }
    return false;
}

cudaError_t launch(const void* fn, dim3 grid, dim3 block, void** args, cudaStream_t s)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, fn, args);
}

int status_of(cudaError_t e) { return e == cudaSuccess ? W8_OK : W8_ERR_CUDA; }

// Grid of a row kernel: one CTA per row for few rows; for many rows, the CTAs that fit on
// the GPU at once (occupancy of this kernel at this block size, cached), each looping over
// rows.
unsigned row_grid(const void* fn, int threads, int M)
{
    if (M < kManyRows) return (unsigned)M;
    int sms = 0;
    if (check_device(&sms) != W8_OK || sms <= 0) return (unsigned)M;
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, int> cache;
    int per = 0;
    {
        std::lock_guard<std::mutex> lk(mu);
        auto it = cache.find({fn, threads});
        if (it != cache.end()) per = it->second;
    }
    if (per == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, fn, threads, 0) != cudaSuccess || per < 1) per = 1;
        std::lock_guard<std::mutex> lk(mu);
        cache[{fn, threads}] = per;
    }
    const long long g = (long long)sms * per;
    return (unsigned)(g < M ? g : M);
}

}  // namespace

int launch_quant_rows(int qfmt, const void* x, int M, int K, int ldx, void* q, float* scale, cudaStream_t s)
{
    int threads, cpt;
    if (!row_shape(M, K / 8, &threads, &cpt)) return W8_ERR_UNSUPPORTED;
    const __nv_bfloat16* xp = static_cast<const __nv_bfloat16*>(x);
    uint8_t* qp = static_cast<uint8_t*>(q);
    void* args[] = {(void*)&xp, (void*)&M, (void*)&K, (void*)&ldx, (void*)&qp, (void*)&scale};
    const void* fn = nullptr;
    if (qfmt == W8_Q_FP8)
        fn = cpt == 1 ? (const void*)quant_rows_kernel<W8_Q_FP8, 1>
                      : cpt == 2 ? (const void*)quant_rows_kernel<W8_Q_FP8, 2> : (const void*)quant_rows_kernel<W8_Q_FP8, 4>;
    else
        fn = cpt == 1 ? (const void*)quant_rows_kernel<W8_Q_INT8, 1>
                      : cpt == 2 ? (const void*)quant_rows_kernel<W8_Q_INT8, 2>
                                 : (const void*)quant_rows_kernel<W8_Q_INT8, 4>;
    return status_of(launch(fn, dim3(row_grid(fn, threads, M)), dim3(threads), args, s));
}

int launch_quant_group128(const void* x, int M, int K, int ldx, void* q, float* scale, int ue8m0, cudaStream_t s)
{
    const long long threads = (long long)M * (K / 128) * 16;
    const long long blocks = (threads + 255) / 256;
    if (blocks > 0x7FFFFFFF) return W8_ERR_UNSUPPORTED;
    const __nv_bfloat16* xp = static_cast<const __nv_bfloat16*>(x);
    uint8_t* qp = static_cast<uint8_t*>(q);
    void* args[] = {(void*)&xp, (void*)&M, (void*)&K, (void*)&ldx, (void*)&qp, (void*)&scale, (void*)&ue8m0};
    return status_of(launch((const void*)quant_group128_kernel, dim3((unsigned)blocks), dim3(256), args, s));
}

int launch_quant_weight_block(const void* w, int N, int K, void* q, float* scale, int ue8m0, cudaStream_t s)
{
    const __nv_bfloat16* wp = static_cast<const __nv_bfloat16*>(w);
    uint8_t* qp = static_cast<uint8_t*>(q);
    void* args[] = {(void*)&wp, (void*)&N, (void*)&K, (void*)&qp, (void*)&scale, (void*)&ue8m0};
    dim3 grid((K + 127) / 128, (N + 127) / 128);
    if (grid.y > 65535) return W8_ERR_UNSUPPORTED;
    return status_of(launch((const void*)quant_weight_block_kernel, grid, dim3(256), args, s));
}

int launch_rmsnorm_quant(const void* x, const void* gamma, float eps, int M, int H, int ldx, void* q, float* scale,
                         int group, int ue8m0, cudaStream_t s)
{
    int threads, cpt;
    if (!row_shape(M, H / 8, &threads, &cpt)) return W8_ERR_UNSUPPORTED;
    const __nv_bfloat16* xp = static_cast<const __nv_bfloat16*>(x);
    const __nv_bfloat16* gp = static_cast<const __nv_bfloat16*>(gamma);
    uint8_t* qp = static_cast<uint8_t*>(q);
    void* args[] = {(void*)&xp, (void*)&gp, (void*)&eps, (void*)&M, (void*)&H, (void*)&ldx, (void*)&qp, (void*)&scale,
                    (void*)&ue8m0};
    const void* fn;
    if (group)
        fn = cpt == 1 ? (const void*)rmsnorm_quant_kernel<1, true>
                      : cpt == 2 ? (const void*)rmsnorm_quant_kernel<2, true> : (const void*)rmsnorm_quant_kernel<4, true>;
    else
        fn = cpt == 1 ? (const void*)rmsnorm_quant_kernel<1, false>
                      : cpt == 2 ? (const void*)rmsnorm_quant_kernel<2, false> : (const void*)rmsnorm_quant_kernel<4, false>;
    return status_of(launch(fn, dim3(M), dim3(threads), args, s));
}

int launch_silu_mul_quant(const void* xgu, int M, int I, int ld, void* q, float* scale, int group, int ue8m0,
                          cudaStream_t s)
{
    int threads, cpt;
    if (!row_shape(M, I / 8, &threads, &cpt)) return W8_ERR_UNSUPPORTED;
    const __nv_bfloat16* xp = static_cast<const __nv_bfloat16*>(xgu);
    uint8_t* qp = static_cast<uint8_t*>(q);
    void* args[] = {(void*)&xp, (void*)&M, (void*)&I, (void*)&ld, (void*)&qp, (void*)&scale, (void*)&ue8m0};
    const void* fn;
    if (group)
        fn = cpt == 1 ? (const void*)silu_mul_quant_kernel<1, true>
                      : cpt == 2 ? (const void*)silu_mul_quant_kernel<2, true> : (const void*)silu_mul_quant_kernel<4, true>;
    else
        fn = cpt == 1 ? (const void*)silu_mul_quant_kernel<1, false>
                      : cpt == 2 ? (const void*)silu_mul_quant_kernel<2, false> : (const void*)silu_mul_quant_kernel<4, false>;
    return status_of(launch(fn, dim3(M), dim3(threads), args, s));
}

}  // namespace w8
