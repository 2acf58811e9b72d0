// w8_qknr.cu -- query/key rms_norm + rotary embedding on the merged qkv projection
// ("PyTorch integra Helion en vLLM para acelerar inferencia FP8", section "Kernels
// Helion implementados": fused_qk_norm_rope; the page names the kernel, no formula).
//
// For qkv[T, (Hq + 2 Hkv) * D] bf16 (query heads, key heads, value heads; D values each)
// and every token t and query or key head:
//   y_k = (x_k * r) * w_k,  r = 1 / sqrt(ss / D + eps),  ss = sum x_k^2 (fp64, then fp32),
//   w = the query or key head-dimension weight;
//   with c_i, s_i the cosine / sine row of the token's position (table input,
//   fp32 [max_pos, D]: cosines then sines), each pair (y_i, y_{i+D/2}) is rotated:
//   o_i = y_i c_i - y_{i+D/2} s_i,  o_{i+D/2} = y_{i+D/2} c_i + y_i s_i  (fp32), -> bf16.
// Value heads are copied (or left in place).  One warp per (token, head); lane l holds
// the D/64 consecutive elements l*D/64.. of each half, so every rotated pair is in one
// thread.  HBM-bound: each head is read once and written once.
#include <cuda_bf16.h>

#include "w8_internal.h"
#include "w8_ptx.cuh"

namespace w8 {
namespace {

static __device__ int g_qknr_status;

template <int C>   // elements per lane per half (D = 64 C)
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
    const long long wid = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (wid >= (long long)T * H) return;
    const int lane = threadIdx.x & 31;
    const int t = (int)(wid / H), h = (int)(wid % H);
    const __nv_bfloat16* x = qkv + (size_t)wid * D;
    __nv_bfloat16* o = out + (size_t)wid * D;
    float lo[C], hi[C];
#pragma unroll
    for (int j = 0; j < C; ++j) {
        lo[j] = __bfloat162float(x[lane * C + j]);
        hi[j] = __bfloat162float(x[HALF + lane * C + j]);
    }
    if (h >= Hq + Hkv) {
        // value head: pass through
        if (o != x)
#pragma unroll
            for (int j = 0; j < C; ++j) {
                o[lane * C + j] = x[lane * C + j];
                o[HALF + lane * C + j] = x[HALF + lane * C + j];
            }
        return;
    }
    const long long p = positions[t];
    if (p < 0 || p >= max_pos) {
        if (lane == 0) atomicCAS(&g_qknr_status, 0, W8_ERR_INVALID_ARG);
        return;
    }
    // sum of squares: each square of a bf16 is exact in fp64; lane sums, then a fixed tree
    double ss = 0.0;
#pragma unroll
    for (int j = 0; j < C; ++j) {
        ss = __fma_rn((double)lo[j], (double)lo[j], ss);
        ss = __fma_rn((double)hi[j], (double)hi[j], ss);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, off);
    const float mean = __fdiv_rn(__double2float_rn(ss), (float)D);
    const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(mean, eps)));
    const __nv_bfloat16* w = (h < Hq) ? qw : kw;
    const float* cs = cos_sin + (size_t)p * D;
#pragma unroll
    for (int j = 0; j < C; ++j) {
        const int i = lane * C + j;
        const float yl = __fmul_rn(__fmul_rn(lo[j], r), __bfloat162float(w[i]));
        const float yh = __fmul_rn(__fmul_rn(hi[j], r), __bfloat162float(w[HALF + i]));
        const float c = __ldg(cs + i), s = __ldg(cs + HALF + i);
        o[i] = __float2bfloat16_rn(__fsub_rn(__fmul_rn(yl, c), __fmul_rn(yh, s)));
        o[HALF + i] = __float2bfloat16_rn(__fadd_rn(__fmul_rn(yh, c), __fmul_rn(yl, s)));
    }
}

}  // namespace

int launch_qk_norm_rope(const void* qkv, void* out, int T, int Hq, int Hkv, int D, const void* q_weight,
                        const void* k_weight, const float* cos_sin, int max_pos, const long long* positions, float eps,
                        cudaStream_t s)
{
    const long long warps = (long long)T * (Hq + 2 * Hkv);
    if (warps == 0) return W8_OK;
    const long long blocks = (warps + 3) / 4;
    if (blocks > 0x7FFFFFFF) return W8_ERR_UNSUPPORTED;
    const void* fn = D == 64 ? (const void*)qk_norm_rope_kernel<1>
                   : D == 128 ? (const void*)qk_norm_rope_kernel<2> : (const void*)qk_norm_rope_kernel<4>;
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
