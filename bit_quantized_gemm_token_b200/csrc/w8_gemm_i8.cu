// w8_gemm_i8.cu -- kernel instantiations: W8A8-INT8 (s8 x s8 -> s32), 128-row MMA tile, every weight tile width.
#include "w8_gemm_kernel.cuh"

namespace w8 {
namespace gemm {
namespace {

template <int BN>
cudaError_t launch_kps(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s)
{
    return p.kps == 2 ? launch_one<128, BN, KIND_I8, false, 2>(p, m, a, s)
                      : launch_one<128, BN, KIND_I8, false, 1>(p, m, a, s);
}

}  // namespace

cudaError_t launch_i8(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s)
{
    switch (p.bn) {
    case 16: return launch_kps<16>(p, m, a, s);
    case 32: return launch_kps<32>(p, m, a, s);
    case 64: return launch_kps<64>(p, m, a, s);
    case 128: return launch_kps<128>(p, m, a, s);
    case 256: return launch_kps<256>(p, m, a, s);
    default: return cudaErrorNotSupported;
    }
}

int status_i8(int clear) { return status_word(clear); }

}  // namespace gemm
}  // namespace w8
