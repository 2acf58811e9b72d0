// w8_noalloc.cu -- w8_gemm for callers that cannot allocate device memory.
//
// Some callers have no way to provide the Split-K workspace: code that runs inside a
// framework whose allocator they do not own (a plugin, a custom operator in a runtime
// that forbids cudaMalloc while serving), or code that must not allocate at all after
// start-up (a latency-critical service, a memory budget fixed at load time).  For them
// w8_gemm_noalloc uses a scratch area that belongs to the library's device code: the
// file-scope array below.  Every GPU that uses it holds it until the process exits.
//
// When the array reaches the device: with eager module loading, when the library's
// device code is loaded; with lazy module loading (CUDA_MODULE_LOADING=LAZY, the
// default of recent CUDA releases), when its address is first asked for.  That happens
// in the first call on each device, whatever variant that call resolves to, so one
// warm-up call before a memory budget is fixed (or before a stream capture) settles it.
//
// The array is shared by every call on a device and keeps what the last call left in
// it; the ticket counters a call uses are cleared at the start of that call.  Calls
// that overlap on the GPU (for example on two streams at once) race on it.
#include <mutex>

#include "w8_internal.h"

namespace w8 {
namespace {

// Largest scratch a call may need: the fixed ticket-counter area plus the partial
// slots of the chosen variant.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};   // device address of the array, per device (set up once)

// The array's name is only a host-side stand-in; the device address comes from the
// runtime, once per device, with that device current.
int noalloc_scratch(void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return W8_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return W8_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return W8_OK;
}

}  // namespace
}  // namespace w8

using namespace w8;

extern "C" int w8_gemm_noalloc(int fmt, const void* A_q, const float* A_scale, const void* W_q,
                               const float* W_scale, void* out, int M, int N, int K, int variant,
                               w8_stream_t stream)
{
    if (!A_q || !W_q || !out || !A_scale || !W_scale) return W8_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0) return W8_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(A_q) & 15) || (reinterpret_cast<uintptr_t>(W_q) & 15) ||
        (reinterpret_cast<uintptr_t>(out) & 1))
        return W8_ERR_ALIGNMENT;
    int sms = 0;
    int rc = check_device(&sms);
    if (rc != W8_OK) return rc;
    // the same variant resolution as w8_gemm: per-shape table, then the built-in rule
    int v = w8_gemm_resolve_variant(fmt, M, N, K, variant);
    if (v < 0) return v;
    GemmPlan plan;
    rc = gemm_plan(fmt, M, N, K, v, sms, &plan);
    if (rc != W8_OK) return rc;
    if (plan.ws_bytes > kNoAllocScratchBytes) return W8_ERR_WORKSPACE;   // beyond the fixed maximum
    // the address is looked up on every device's first call, whether or not this call
    // needs scratch, so that the array is in place after any first call
    void* scratch = nullptr;
    rc = noalloc_scratch(&scratch);
    if (rc != W8_OK) return rc;
    if (plan.ws_bytes > 0) {
        // counters of this call's tiles must start at zero
        cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
        if (cudaMemsetAsync(scratch, 0, (size_t)plan.tiles * 4, s) != cudaSuccess) return W8_ERR_CUDA;
    } else {
        scratch = nullptr;
    }
    return gemm_launch(plan, A_q, A_scale, W_q, W_scale, out, nullptr, scratch, kNoAllocScratchBytes,
                       reinterpret_cast<cudaStream_t>(stream));
}
