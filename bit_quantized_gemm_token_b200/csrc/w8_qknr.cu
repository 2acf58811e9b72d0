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
// Value heads are copied (or left in place).  One warp per four consecutive heads of a
// token (their loads issued together); lane l holds the D/64 consecutive elements
// l*D/64.. of each half of every head, so every rotated pair is in one thread.  HBM-bound:
// each head is read once and written once.
#include <cuda_bf16.h>

#include <type_traits>

#include "w8_internal.h"
#include "w8_ptx.cuh"
#include "w8_sumsq.cuh"

namespace w8 {
namespace {

static __device__ int g_qknr_status;

// C = elements per lane per half (D = 64 C); HPW = heads per warp (one token's
// consecutive heads: their loads are all in flight together, and the token's cos / sin
// values are loaded once for them)
template <int C, int HPW>
__global__ void __launch_bounds__(128) qk_norm_rope_kernel(const __nv_bfloat16* __restrict__ qkv,
                                                           __nv_bfloat16* __restrict__ out, int T, int Hq, int Hkv,
                                                           const __nv_bfloat16* __restrict__ qw,
                                                           const __nv_bfloat16* __restrict__ kw,
                                                           const float* __restrict__ cos_sin, int max_pos,
                                                           const long long* __restrict__ positions, float eps)
{
    ptx::grid_dep_launch();
    ptx::grid_dep_wait();
    constexpr int D = 64 * C, HALF = 32 * C;
    const int H = Hq + 2 * Hkv;
    const int groups = (H + HPW - 1) / HPW;
    const long long wid = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (wid >= (long long)T * groups) return;
    const int lane = threadIdx.x & 31;
    const int t = (int)(wid / groups), h0 = (int)(wid % groups) * HPW;
    const int nh = min(HPW, H - h0);
    // lane l: elements [l*C, l*C + C) of each half, as one C*2-byte vector
    using Vec = typename std::conditional<C == 1, unsigned short, typename std::conditional<C == 2, unsigned int, uint2>::type>::type;
    Vec lov[HPW], hiv[HPW];
#pragma unroll
    for (int j = 0; j < HPW; ++j) {
        if (j < nh) {
            const __nv_bfloat16* x = qkv + ((size_t)t * H + h0 + j) * D;
            lov[j] = *reinterpret_cast<const Vec*>(x + lane * C);
            hiv[j] = *reinterpret_cast<const Vec*>(x + HALF + lane * C);
        }
    }
    const long long p = positions[t];
    const bool pos_ok = p >= 0 && p < max_pos;
    float cv[C], sv[C];
    if (pos_ok && h0 < Hq + Hkv) {
        const float* cs = cos_sin + (size_t)p * D;
#pragma unroll
        for (int i = 0; i < C; ++i) {
            cv[i] = __ldg(cs + lane * C + i);
            sv[i] = __ldg(cs + HALF + lane * C + i);
        }
    }
    if (!pos_ok && h0 < Hq + Hkv && lane == 0) atomicCAS(&g_qknr_status, 0, W8_ERR_INVALID_ARG);
    auto unpack = [](Vec v, float (&f)[C]) {
        const unsigned short* b = reinterpret_cast<const unsigned short*>(&v);
#pragma unroll
        for (int i = 0; i < C; ++i) f[i] = __uint_as_float((uint32_t)b[i] << 16);
    };
#pragma unroll
    for (int j = 0; j < HPW; ++j) {
        if (j >= nh) break;
        const int h = h0 + j;
        __nv_bfloat16* o = out + ((size_t)t * H + h) * D;
        if (h >= Hq + Hkv) {
            // value head: pass through
            if (out != qkv) {
                *reinterpret_cast<Vec*>(o + lane * C) = lov[j];
                *reinterpret_cast<Vec*>(o + HALF + lane * C) = hiv[j];
            }
            continue;
        }
        if (!pos_ok) continue;
        float lo[C], hi[C];
        unpack(lov[j], lo);
        unpack(hiv[j], hi);
        // the exact sum of squares rounded once to fp32 (w8_sumsq.cuh): lane sums, then the warp
        DSum ss{0.0, 0.0};
#pragma unroll
        for (int i = 0; i < C; ++i) {
            ss = dsum_sq(ss, lo[i]);
            ss = dsum_sq(ss, hi[i]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss = dsum_add(ss, dsum_shfl_xor(ss, off));
        const float mean = __fdiv_rn(dsum_to_f32(ss), (float)D);
        const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(mean, eps)));
        const __nv_bfloat16* w = (h < Hq) ? qw : kw;
        float wl[C], wh[C];
        unpack(*reinterpret_cast<const Vec*>(w + lane * C), wl);
        unpack(*reinterpret_cast<const Vec*>(w + HALF + lane * C), wh);
        unsigned short ol[C], oh[C];
#pragma unroll
        for (int i = 0; i < C; ++i) {
            const float yl = __fmul_rn(__fmul_rn(lo[i], r), wl[i]);
            const float yh = __fmul_rn(__fmul_rn(hi[i], r), wh[i]);
            const __nv_bfloat16 a = __float2bfloat16_rn(__fsub_rn(__fmul_rn(yl, cv[i]), __fmul_rn(yh, sv[i])));
            const __nv_bfloat16 b = __float2bfloat16_rn(__fadd_rn(__fmul_rn(yh, cv[i]), __fmul_rn(yl, sv[i])));
            ol[i] = *reinterpret_cast<const unsigned short*>(&a);
            oh[i] = *reinterpret_cast<const unsigned short*>(&b);
        }
        *reinterpret_cast<Vec*>(o + lane * C) = *reinterpret_cast<const Vec*>(ol);
        *reinterpret_cast<Vec*>(o + HALF + lane * C) = *reinterpret_cast<const Vec*>(oh);
    }
}

}  // namespace

int launch_qk_norm_rope(const void* qkv, void* out, int T, int Hq, int Hkv, int D, const void* q_weight,
                        const void* k_weight, const float* cos_sin, int max_pos, const long long* positions, float eps,
                        cudaStream_t s)
{
    constexpr int kHeadsPerWarp = 4;
    const long long warps = (long long)T * ((Hq + 2 * Hkv + kHeadsPerWarp - 1) / kHeadsPerWarp);
    if (warps == 0) return W8_OK;
    const long long blocks = (warps + 3) / 4;
    if (blocks > 0x7FFFFFFF) return W8_ERR_UNSUPPORTED;
    const void* fn = D == 64 ? (const void*)qk_norm_rope_kernel<1, kHeadsPerWarp>
                   : D == 128 ? (const void*)qk_norm_rope_kernel<2, kHeadsPerWarp>
                              : (const void*)qk_norm_rope_kernel<4, kHeadsPerWarp>;
    const __nv_bfloat16* xp = static_cast<const __nv_bfloat16*>(qkv);
    __nv_bfloat16* op = static_cast<__nv_bfloat16*>(out);
    const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(q_weight);
    const __nv_bfloat16* kp = static_cast<const __nv_bfloat16*>(k_weight);
    void* args[] = {(void*)&xp, (void*)&op, (void*)&T, (void*)&Hq, (void*)&Hkv, (void*)&qp, (void*)&kp,
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
