// w8_gemm_block.cu -- kernel instantiations: Block-FP8 (per-128-K-block promotion in the epilogue), 128-row MMA tile, narrow tiles.
#include "w8_gemm_kernel.cuh"

namespace w8 {
namespace gemm {
namespace {

template <int BN>
cudaError_t launch_kps(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s)
{
    return p.kps == 2 ? launch_one<128, BN, KIND_F8, true, 2>(p, m, a, s)
                      : launch_one<128, BN, KIND_F8, true, 1>(p, m, a, s);
}

}  // namespace

cudaError_t launch_block(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s)
{
    switch (p.bn) {
    case 16: return launch_kps<16>(p, m, a, s);
    case 32: return launch_kps<32>(p, m, a, s);
    case 64: return launch_kps<64>(p, m, a, s);
    default: return cudaErrorNotSupported;
    }
}

int status_block(int clear) { return status_word(clear); }

}  // namespace gemm
}  // namespace w8
