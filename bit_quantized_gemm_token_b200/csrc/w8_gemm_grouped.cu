// w8_gemm_grouped.cu -- kernel instantiations: the grouped (mixture-of-experts) form of the
// Swap-AB GEMM (FP8-dynamic and W8A8-INT8; token tiles of 16, 32 and 64 for decode
// routings, 128 and 256 for prefill routings with hundreds of tokens per expert).
#include "w8_gemm_kernel.cuh"

namespace w8 {
namespace gemm {
namespace {

template <int BN, int KIND>
cudaError_t launch_kps(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s)
{
    return p.kps == 2 ? launch_one<128, BN, KIND, false, 2, false, true>(p, m, a, s)
                      : launch_one<128, BN, KIND, false, 1, false, true>(p, m, a, s);
}

template <int KIND>
cudaError_t launch_bn(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s)
{
    switch (p.bn) {
    case 16: return launch_kps<16, KIND>(p, m, a, s);
    case 32: return launch_kps<32, KIND>(p, m, a, s);
    case 64: return launch_kps<64, KIND>(p, m, a, s);
    case 128: return launch_kps<128, KIND>(p, m, a, s);
    case 256: return launch_kps<256, KIND>(p, m, a, s);
    default: return cudaErrorNotSupported;
    }
}

}  // namespace

cudaError_t launch_grouped(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s)
{
    return p.fmt == W8_FMT_INT8 ? launch_bn<KIND_I8>(p, m, a, s) : launch_bn<KIND_F8>(p, m, a, s);
}

int status_grouped(int clear) { return status_word(clear); }

}  // namespace gemm
}  // namespace w8
