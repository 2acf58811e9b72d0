// w8_qknr.cu -- query/key rms_norm + rotary embedding on the merged qkv projection
// ("PyTorch integra Helion en vLLM para acelerar inferencia FP8", section "Kernels
// Helion implementados": fused_qk_norm_rope; the page names the kernel, no formula).
//
// For qkv[T, (Hq + 2 Hkv) * D] bf16 (query heads, key heads, value heads; D values each)
// and every token t and query or key head:
//   y_k = (x_k * r) * w_k,  r = 1 / sqrt(ss / D + eps),  ss = sum x_k^2 (exact, then fp32),
//   w = the query or key head-dimension weight;
//   with c_i, s_i the cosine / sine row of the token's position (table input,
//   fp32 [max_pos, D]: cosines then sines), each pair (y_i, y_{i+D/2}) is rotated:
//   o_i = y_i c_i - y_{i+D/2} s_i,  o_{i+D/2} = y_{i+D/2} c_i + y_i s_i  (fp32), -> bf16.
// Value heads are copied (or left in place).  D / 16 lanes share a head: lane s of the
// head's group holds the 8 consecutive elements 8s.. of each half (one 16-byte vector per
// half), so every rotated pair is in one thread and a warp covers 512 / D consecutive heads
// of a token at once; each warp takes G such groups, their loads all issued before any
// arithmetic.  HBM-bound: each head is read once and written once.
#include <cuda_bf16.h>

#include "w8_internal.h"
#include "w8_ptx.cuh"
#include "w8_sumsq.cuh"

namespace w8 {
namespace {

static __device__ int g_qknr_status;

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8])
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);   // .x = a (low half), .y = b
    return *reinterpret_cast<const uint32_t*>(&v);
}

// D = head dimension (64, 128 or 256); G = head groups per warp; Hn = heads touched per
// token (query + key heads in place, all heads otherwise); units = T * ceil(Hn / (512 / D)).
// At most 80 registers (6 CTAs of 128 threads per SM): measured on B200 at 4096 and 16384
// tokens ahead of 64 registers with spills (8 CTAs), 96 (5) and of one or four head
// groups per warp.
template <int D, int G>
__global__ void __launch_bounds__(128, 6) qk_norm_rope_kernel(const __nv_bfloat16* __restrict__ qkv,
                                                           __nv_bfloat16* __restrict__ out, int Hq, int Hkv, int Hn,
                                                           int units, const __nv_bfloat16* __restrict__ qw,
                                                           const __nv_bfloat16* __restrict__ kw,
                                                           const float* __restrict__ cos_sin, int max_pos,
                                                           const long long* __restrict__ positions, float eps)
{
    ptx::grid_dep_launch();
    ptx::grid_dep_wait();
    constexpr int HALF = D / 2, LPH = D / 16, HPW = 32 / LPH;
    // no term passes through more than 16 (the lane's fp64 chain) + log2(LPH) roundings
    constexpr int kDepth = 16 + 5;
    const int H = Hq + 2 * Hkv;
    const int groups = (Hn + HPW - 1) / HPW;
    const int wid = (int)(((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * G);
    if (wid >= units) return;
    const int lane = threadIdx.x & 31, sub = lane % LPH;
    uint4 lov[G], hiv[G];
    int tt[G], hh[G];
    bool act[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const int u = wid + g;
        tt[g] = u / groups;
        hh[g] = (u - tt[g] * groups) * HPW + lane / LPH;
        act[g] = u < units && hh[g] < Hn;
        if (act[g]) {
            const __nv_bfloat16* x = qkv + ((size_t)tt[g] * H + hh[g]) * D + sub * 8;
            lov[g] = *reinterpret_cast<const uint4*>(x);
            hiv[g] = *reinterpret_cast<const uint4*>(x + HALF);
        } else {
            lov[g] = make_uint4(0, 0, 0, 0);
            hiv[g] = make_uint4(0, 0, 0, 0);
        }
    }
    long long pos[G];
#pragma unroll
    for (int g = 0; g < G; ++g) pos[g] = act[g] && hh[g] < Hq + Hkv ? __ldg(positions + tt[g]) : 0;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const int h = hh[g];
        const bool rot = act[g] && h < Hq + Hkv;
        const bool pos_ok = pos[g] >= 0 && pos[g] < max_pos;
        if (rot && !pos_ok && sub == 0) atomicCAS(&g_qknr_status, 0, W8_ERR_INVALID_ARG);
        __nv_bfloat16* o = out + ((size_t)tt[g] * H + h) * D + sub * 8;
        if (act[g] && !rot && out != qkv) {
            // value head: pass through
            *reinterpret_cast<uint4*>(o) = lov[g];
            *reinterpret_cast<uint4*>(o + HALF) = hiv[g];
        }
        float lo[8], hi[8];
        unpack8(lov[g], lo);
        unpack8(hiv[g], hi);
        // the exact sum of squares of the head, rounded once to fp32 (w8_sumsq.cuh); every
        // lane of the warp runs the butterflies (inactive lanes hold zeros)
        double ss64 = 0.0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            ss64 = __fma_rn((double)lo[i], (double)lo[i], ss64);
            ss64 = __fma_rn((double)hi[i], (double)hi[i], ss64);
        }
#pragma unroll
        for (int off = LPH / 2; off > 0; off >>= 1) ss64 = __dadd_rn(ss64, __shfl_xor_sync(0xFFFFFFFFu, ss64, off));
        float ssf;
        const bool sure = sq_round_certain(ss64, kDepth, &ssf);
        if (__any_sync(0xFFFFFFFFu, !sure)) {
            DSum ds{0.0, 0.0};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                ds = dsum_sq(ds, lo[i]);
                ds = dsum_sq(ds, hi[i]);
            }
#pragma unroll
            for (int off = LPH / 2; off > 0; off >>= 1) ds = dsum_add(ds, dsum_shfl_xor(ds, off));
            if (!sure) ssf = dsum_to_f32(ds);
        }
        if (!rot || !pos_ok) continue;
        const float* cs = cos_sin + (size_t)pos[g] * D + sub * 8;
        const float4 c0 = __ldg(reinterpret_cast<const float4*>(cs));
        const float4 c1 = __ldg(reinterpret_cast<const float4*>(cs + 4));
        const float4 s0 = __ldg(reinterpret_cast<const float4*>(cs + HALF));
        const float4 s1 = __ldg(reinterpret_cast<const float4*>(cs + HALF + 4));
        const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        // ss / D with D a power of two is an exact scaling (the same rounding as the quotient)
        const float mean = __fmul_rn(ssf, 1.0f / D);
        const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(mean, eps)));
        const __nv_bfloat16* w = (h < Hq ? qw : kw) + sub * 8;
        float wl[8], wh[8];
        unpack8(__ldg(reinterpret_cast<const uint4*>(w)), wl);
        unpack8(__ldg(reinterpret_cast<const uint4*>(w + HALF)), wh);
        uint32_t ol[4], oh[4];
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            float a[2], b[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const float yl = __fmul_rn(__fmul_rn(lo[i + k], r), wl[i + k]);
                const float yh = __fmul_rn(__fmul_rn(hi[i + k], r), wh[i + k]);
                a[k] = __fsub_rn(__fmul_rn(yl, cv[i + k]), __fmul_rn(yh, sv[i + k]));
                b[k] = __fadd_rn(__fmul_rn(yh, cv[i + k]), __fmul_rn(yl, sv[i + k]));
            }
            ol[i / 2] = pack_bf16x2(a[0], a[1]);
            oh[i / 2] = pack_bf16x2(b[0], b[1]);
        }
        *reinterpret_cast<uint4*>(o) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
        *reinterpret_cast<uint4*>(o + HALF) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
    }
}

template <int D>
const void* qknr_fn()
{
    return (const void*)qk_norm_rope_kernel<D, 2>;
}

}  // namespace

int launch_qk_norm_rope(const void* qkv, void* out, int T, int Hq, int Hkv, int D, const void* q_weight,
                        const void* k_weight, const float* cos_sin, int max_pos, const long long* positions, float eps,
                        cudaStream_t s)
{
    constexpr int kGroupsPerWarp = 2;
    const int Hn = out == qkv ? Hq + Hkv : Hq + 2 * Hkv;
    const int hpw = 512 / D;
    const long long units = (long long)T * ((Hn + hpw - 1) / hpw);
    if (units == 0) return W8_OK;
    if (units > 0x7FFFFFFFLL - 256) return W8_ERR_UNSUPPORTED;
    const long long warps = (units + kGroupsPerWarp - 1) / kGroupsPerWarp;
    const long long blocks = (warps + 3) / 4;
    const void* fn = D == 64 ? qknr_fn<64>() : D == 128 ? qknr_fn<128>() : qknr_fn<256>();
    const __nv_bfloat16* xp = static_cast<const __nv_bfloat16*>(qkv);
    __nv_bfloat16* op = static_cast<__nv_bfloat16*>(out);
    const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(q_weight);
    const __nv_bfloat16* kp = static_cast<const __nv_bfloat16*>(k_weight);
    int un = (int)units;
    void* args[] = {(void*)&xp, (void*)&op, (void*)&Hq, (void*)&Hkv, (void*)&Hn, (void*)&un, (void*)&qp, (void*)&kp,
                    (void*)&cos_sin, (void*)&max_pos, (void*)&positions, (void*)&eps};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(128);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, fn, args) == cudaSuccess ? W8_OK : W8_ERR_CUDA;
}

int qknr_device_status(int clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_qknr_status, sizeof(int)) != cudaSuccess) return W8_ERR_CUDA;
    if (clear && v != 0) {
        const int z = 0;
        if (cudaMemcpyToSymbol(g_qknr_status, &z, sizeof(int)) != cudaSuccess) return W8_ERR_CUDA;
    }
    return v;
}

}  // namespace w8
