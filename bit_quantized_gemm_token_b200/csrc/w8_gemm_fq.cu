// w8_gemm_fq.cu -- kernel instantiations: the GEMM with fused activation quantization
// (Swap-AB; FP8-dynamic and W8A8-INT8 per token, Block-FP8 per 1 x 128 group), token
// tiles of 16, 32 and 64.
#include "w8_gemm_kernel.cuh"

namespace w8 {
namespace gemm {
namespace {

template <int BN, int KIND, bool BLOCK>
cudaError_t launch_kps(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s)
{
    return p.kps == 2 ? launch_one<128, BN, KIND, BLOCK, 2, true>(p, m, a, s)
                      : launch_one<128, BN, KIND, BLOCK, 1, true>(p, m, a, s);
}

template <int KIND, bool BLOCK>
cudaError_t launch_bn(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s)
{
    switch (p.bn) {
    case 16: return launch_kps<16, KIND, BLOCK>(p, m, a, s);
    case 32: return launch_kps<32, KIND, BLOCK>(p, m, a, s);
    case 64: return launch_kps<64, KIND, BLOCK>(p, m, a, s);
    default: return cudaErrorNotSupported;
    }
}

}  // namespace

cudaError_t launch_fq(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s)
{
    if (p.fmt >= W8_FMT_BLOCK_FP8) return launch_bn<KIND_F8, true>(p, m, a, s);
    if (p.fmt == W8_FMT_INT8) return launch_bn<KIND_I8, false>(p, m, a, s);
    return launch_bn<KIND_F8, false>(p, m, a, s);
}

int status_fq(int clear) { return status_word(clear); }

}  // namespace gemm
}  // namespace w8
