// w8_gemm_bm64.cu -- kernel instantiations: Standard form with the 64-row token tile in
// the MMA's M slot and 128- or 256-row weight tiles in its N slot (FP8-dynamic, INT8).
#include "w8_gemm_kernel.cuh"

namespace w8 {
namespace gemm {
namespace {

template <int BN, int KIND>
cudaError_t launch_kps(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s)
{
    return p.kps == 2 ? launch_one<64, BN, KIND, false, 2>(p, m, a, s)
                      : launch_one<64, BN, KIND, false, 1>(p, m, a, s);
}

}  // namespace

cudaError_t launch_bm64(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s)
{
    const bool i8 = p.fmt == W8_FMT_INT8;
    switch (p.bn) {
    case 128: return i8 ? launch_kps<128, KIND_I8>(p, m, a, s) : launch_kps<128, KIND_F8>(p, m, a, s);
    case 256: return i8 ? launch_kps<256, KIND_I8>(p, m, a, s) : launch_kps<256, KIND_F8>(p, m, a, s);
    default: return cudaErrorNotSupported;
    }
}

int status_bm64(int clear) { return status_word(clear); }

}  // namespace gemm
}  // namespace w8
