// w8_api.cu -- the C ABI (include/w8.h): argument validation, device check, variant
// resolution (per-shape table, then a built-in rule) and dispatch to the kernels.
// Nothing here allocates device memory or synchronises.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "w8_internal.h"

namespace w8 {
namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

struct DevInfo {
    bool probed = false;
    bool ok = false;
    int sms = 0;
};

std::mutex g_dev_mu;
DevInfo g_dev[64];

// ---- per-shape table ----------------------------------------------------------------
struct Entry {
    int fmt, N, K, m_max, variant;
};
std::mutex g_tab_mu;
std::vector<Entry> g_table;

}  // namespace

int check_device(int* sm_count)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return W8_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DevInfo& d = g_dev[dev];
    if (!d.probed) {
        d.probed = true;
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) {
            d.ok = (major == 10 && minor == 0);
            d.sms = sms;
        }
    }
    if (!d.ok) return W8_ERR_NO_DEVICE;
    if (sm_count) *sm_count = d.sms;
    return W8_OK;
}

int table_lookup(int fmt, int N, int K, int M)
{
    std::lock_guard<std::mutex> lk(g_tab_mu);
    const Entry* best = nullptr;
    for (const Entry& e : g_table)
        if (e.fmt == fmt && e.N == N && e.K == K && e.m_max >= M && (!best || e.m_max < best->m_max)) best = &e;
    return best ? best->variant : 0;
}

namespace {

// Built-in rule when the table has no entry: the decode form for FP8 / INT8 up to 64
// tokens; Swap-AB with the narrowest token tile and the balanced partition for Block-FP8
// decode sizes; CTA-pair (FP8 / INT8) or Standard (Block-FP8) whole tiles for prefill.
// Grouped GEMM default: Swap-AB over the balanced partition with the narrowest token tile
// that holds an expert's largest token count (64 beyond that: several token tiles, two
// CTAs per SM).
int grouped_variant(int max_m)
{
    const int tile = max_m <= 16 ? kTileBN16 : max_m <= 32 ? kTileBN32 : kTileBN64;
    // past 64 tokens per expert (prefill routings): two CTAs per SM, measured 353 against
    // 455 us for 128 experts of 1536 x 2048 at 4096 tokens x top-8 on B200 (128- and
    // 256-token tiles were no faster, or slower)
    if (max_m > 64) return W8_VARIANT(1, 0, tile, 1) | (2 << W8_V_CPS_SHIFT);
    return W8_VARIANT(1, 0, tile, 1);
}

// Decode form for FP8-dynamic / INT8 at M <= 64: the (weight tile, K chunks) pair with
// the lowest estimated time on `sms` SMs.  The estimate (microseconds) is the slowest of
// the HBM stream (~6.5 TB/s), one CTA's stream (~54 GB/s: ~108 KB in flight per SM over
// ~2 us of latency under load) and its chain of tensor-core instructions (~0.084 us per
// 64 x BN x 32 MMA), plus ~0.25 us per K chunk for the exchange in distributed shared
// memory -- the costs measured on B200 for the decode shapes.  0 when none is legal.
int decode_builtin(int fmt, int M, int N, int K, int sms)
{
    const int kbs = (K + 127) / 128;
    double best_t = 1e30;
    int best = 0, best_g = 0;
    for (int bn = 256; bn >= 64; bn -= 16) {
        const int tiles = (N + bn - 1) / bn;
        for (int c = 1; c <= 8 && c <= kbs; ++c) {
            const int g = tiles * c;
            if (g > sms) break;
            const int kb = (kbs + c - 1) / c;
            const double t_hbm = (double)N * K / 6.5e6;
            const double t_cta = (double)bn * kb * 128 / 54e3;
            const double t_mma = kb * 4 * 0.084;
            const double t = std::max(t_hbm, std::max(t_cta, t_mma)) + (c > 1 ? 0.25 * c : 0.0);
            // ties: the launch with more CTAs (more requests in flight)
            if (t < best_t - 1e-9 || (t < best_t + 1e-9 && g > best_g)) {
                const int v = W8_V_EXPLICIT | W8_V_DECODE | ((c - 1) << W8_V_SPLIT_SHIFT) | ((bn / 16 - 1) << W8_V_TILE_SHIFT);
                GemmPlan plan;
                if (gemm_plan(fmt, M, N, K, v, sms, &plan) != W8_OK) continue;
                best_t = t;
                best = v;
                best_g = g;
            }
        }
    }
    return best;
}

int builtin_variant(int fmt, int M, int N, int K, int sms)
{
    const bool block = fmt >= W8_FMT_BLOCK_FP8;
    if (!block && M <= 64) {
        const int v = decode_builtin(fmt, M, N, K, sms);
        if (v) return v;
    }
    if (M <= 16) return W8_VARIANT(1, 0, kTileBN16, 1);
    if (M <= 32) return W8_VARIANT(1, 0, kTileBN32, 1);
    if (M <= 64) return W8_VARIANT(1, 0, kTileBN64, 1);
    // prefill: tensor-bound; every MMA costs about the same issue time whatever its N, so
    // the widest weight tile (256; 64 for Block-FP8, whose promotion keeps the tile in
    // registers) over whole-tile loops.  FP8 / INT8: 256 x 256 tiles on CTA pairs, a
    // third less shared-memory traffic per MMA, hence deeper pipelines (1.71 -> 2.36
    // PFLOP/s on B200 at M = 4096, K = 4096, N = 24576); measured ahead of the one-CTA
    // loops and of Swap-AB from M = 72 on (2x over the four dense shapes at M = 96)
    if (block) return W8_VARIANT(0, 0, kTileBN64, 1);
    return W8_VARIANT(0, 0, kTileBN256, 0) | W8_V_PAIR;
}

int resolve(int fmt, int M, int N, int K, int variant, int sms, GemmPlan* plan)
{
    int v = variant;
    if (!(v & W8_V_EXPLICIT)) {
        const int pdl = v & W8_V_PDL;   // AUTO may still ask for PDL
        v = table_lookup(fmt, N, K, M);
        if (!v) v = builtin_variant(fmt, M, N, K, sms);
        v |= pdl;
    }
    const int rc = gemm_plan(fmt, M, N, K, v, sms, plan);
    return rc == W8_OK ? v : rc;
}

int gemm_common(int fmt, const void* A_q, const float* A_scale, const void* W_q, const float* W_scale, void* out,
                int32_t* out_i32, int M, int N, int K, int variant, void* workspace, size_t ws_bytes,
                cudaStream_t s)
{
    if (!A_q || !W_q || (!out && !out_i32)) return W8_ERR_INVALID_ARG;
    if (!out_i32 && (!A_scale || !W_scale)) return W8_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0) return W8_ERR_INVALID_ARG;
    if (!aligned(A_q, 16) || !aligned(W_q, 16)) return W8_ERR_ALIGNMENT;
    if (out && !aligned(out, 2)) return W8_ERR_ALIGNMENT;
    if (out_i32 && !aligned(out_i32, 4)) return W8_ERR_ALIGNMENT;
    int sms = 0;
    int rc = check_device(&sms);
    if (rc != W8_OK) return rc;
    GemmPlan plan;
    rc = resolve(fmt, M, N, K, variant, sms, &plan);
    if (rc < 0) return rc;
    return gemm_launch(plan, A_q, A_scale, W_q, W_scale, out, out_i32, workspace, ws_bytes, s);
}

size_t round256(size_t n) { return (n + 255) & ~(size_t)255; }

// Workspace of w8_linear: the GEMM's, then (two-kernel path) the codes and the scales.
// The codes never start inside the counter area, even for a GEMM that uses no counters:
// other calls sharing the workspace keep their tile counters there.
size_t linear_codes_offset(const GemmPlan& p)
{
    const size_t counters = (size_t)kMaxCounterTiles * 4;
    return round256(p.ws_bytes > counters ? p.ws_bytes : counters);
}

size_t linear_ws(const GemmPlan& p)
{
    const bool block = p.fmt >= W8_FMT_BLOCK_FP8;
    return linear_codes_offset(p) + round256((size_t)p.M * p.K) + round256((size_t)p.M * (block ? p.kbs : 1) * 4);
}

int linear_common(int fmt, const void* x, int ldx, const void* W_q, const float* W_scale, void* out, int M, int N,
                  int K, int variant, void* workspace, size_t ws_bytes, uint8_t* dbg_q, float* dbg_s, cudaStream_t s)
{
    if (!x || !W_q || !W_scale || !out) return W8_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0 || ldx < K) return W8_ERR_INVALID_ARG;
    if (fmt < W8_FMT_FP8_DYN || fmt > W8_FMT_BLOCK_FP8_UE8M0) return W8_ERR_INVALID_ARG;
    if (ldx % 8 != 0 || !aligned(x, 16) || !aligned(W_q, 16) || !aligned(out, 2)) return W8_ERR_ALIGNMENT;
    if (dbg_q && !aligned(dbg_q, 16)) return W8_ERR_ALIGNMENT;
    int sms = 0;
    int rc = check_device(&sms);
    if (rc != W8_OK) return rc;
    GemmPlan plan;
    int v = resolve(fmt, M, N, K, variant, sms, &plan);
    if (v < 0) return v;
    // the one-kernel form when asked for (explicitly, or by the table's entry for AUTO)
    const bool fused = (v & W8_V_FUSED) || dbg_q || dbg_s;
    v &= ~W8_V_FUSED;
    if (fused) {
        rc = linear_plan(fmt, M, N, K, v, sms, &plan);
        if (rc != W8_OK) return rc;
        return linear_launch(plan, x, ldx, W_q, W_scale, out, workspace, ws_bytes, dbg_q, dbg_s, s);
    }
    // two kernels: the quantizer into the workspace, then the GEMM
    rc = gemm_plan(fmt, M, N, K, v, sms, &plan);
    if (rc != W8_OK) return rc;
    if (workspace == nullptr || ws_bytes < linear_ws(plan)) return W8_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return W8_ERR_ALIGNMENT;
    const bool block = fmt >= W8_FMT_BLOCK_FP8;
    if (!block && K > kRowMaxK) return W8_ERR_UNSUPPORTED;
    uint8_t* base = static_cast<uint8_t*>(workspace);
    uint8_t* Aq = base + linear_codes_offset(plan);
    float* sA = reinterpret_cast<float*>(Aq + round256((size_t)M * K));
    rc = block ? launch_quant_group128(x, M, K, ldx, Aq, sA, fmt == W8_FMT_BLOCK_FP8_UE8M0, s)
               : launch_quant_rows(fmt == W8_FMT_INT8 ? W8_Q_INT8 : W8_Q_FP8, x, M, K, ldx, Aq, sA, s);
    if (rc != W8_OK) return rc;
    return gemm_launch(plan, Aq, sA, W_q, W_scale, out, nullptr, workspace, ws_bytes, s);
}

bool row_args_ok(const void* x, int M, int K, int ldx, const void* q, const float* scale)
{
    return x && q && scale && M > 0 && K > 0 && ldx >= K;
}

}  // namespace
}  // namespace w8

using namespace w8;

extern "C" {

int w8_quant_per_token(int qfmt, const void* x, int M, int K, int ldx, void* q, float* scale, int group, int ue8m0,
                       w8_stream_t stream)
{
    if (!row_args_ok(x, M, K, ldx, q, scale)) return W8_ERR_INVALID_ARG;
    if (qfmt != W8_Q_FP8 && qfmt != W8_Q_INT8) return W8_ERR_INVALID_ARG;
    if (group != 0 && group != 128) return W8_ERR_UNSUPPORTED;
    if ((group != 0 || ue8m0) && qfmt != W8_Q_FP8) return W8_ERR_UNSUPPORTED;
    if (ue8m0 && group == 0) return W8_ERR_UNSUPPORTED;
    if (K % 8 != 0 || ldx % 8 != 0 || !aligned(x, 16) || !aligned(q, 8) || !aligned(scale, 4))
        return W8_ERR_ALIGNMENT;
    if (group != 0 && K % group != 0) return W8_ERR_UNSUPPORTED;
    if (group == 0 && K > kRowMaxK) return W8_ERR_UNSUPPORTED;
    int rc = check_device(nullptr);
    if (rc != W8_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (group == 0) return launch_quant_rows(qfmt, x, M, K, ldx, q, scale, s);
    return launch_quant_group128(x, M, K, ldx, q, scale, ue8m0, s);
}

int w8_quant_weight_block(const void* w, int N, int K, void* q, float* scale, int ue8m0, w8_stream_t stream)
{
    if (!w || !q || !scale || N <= 0 || K <= 0) return W8_ERR_INVALID_ARG;
    if (K % 8 != 0 || !aligned(w, 16) || !aligned(q, 8) || !aligned(scale, 4)) return W8_ERR_ALIGNMENT;
    int rc = check_device(nullptr);
    if (rc != W8_OK) return rc;
    return launch_quant_weight_block(w, N, K, q, scale, ue8m0, reinterpret_cast<cudaStream_t>(stream));
}

int w8_rmsnorm_quant(const void* x, const void* gamma, float eps, int M, int H, int ldx, void* q, float* scale,
                     w8_stream_t stream)
{
    if (!row_args_ok(x, M, H, ldx, q, scale) || !gamma) return W8_ERR_INVALID_ARG;
    if (!(eps >= 0.0f)) return W8_ERR_INVALID_ARG;
    if (H % 8 != 0 || ldx % 8 != 0 || !aligned(x, 16) || !aligned(gamma, 16) || !aligned(q, 8) || !aligned(scale, 4))
        return W8_ERR_ALIGNMENT;
    if (H > kRowMaxK) return W8_ERR_UNSUPPORTED;
    int rc = check_device(nullptr);
    if (rc != W8_OK) return rc;
    return launch_rmsnorm_quant(x, gamma, eps, M, H, ldx, q, scale, 0, 0, reinterpret_cast<cudaStream_t>(stream));
}

int w8_rmsnorm_quant_group(const void* x, const void* gamma, float eps, int M, int H, int ldx, int group, int ue8m0,
                           void* q, float* scale, w8_stream_t stream)
{
    if (!row_args_ok(x, M, H, ldx, q, scale) || !gamma) return W8_ERR_INVALID_ARG;
    if (!(eps >= 0.0f)) return W8_ERR_INVALID_ARG;
    if (group != 128 || H % group != 0) return W8_ERR_UNSUPPORTED;
    if (ldx % 8 != 0 || !aligned(x, 16) || !aligned(gamma, 16) || !aligned(q, 8) || !aligned(scale, 4))
        return W8_ERR_ALIGNMENT;
    if (H > kRowMaxK) return W8_ERR_UNSUPPORTED;
    int rc = check_device(nullptr);
    if (rc != W8_OK) return rc;
    return launch_rmsnorm_quant(x, gamma, eps, M, H, ldx, q, scale, group, ue8m0, reinterpret_cast<cudaStream_t>(stream));
}

int w8_silu_mul_quant(const void* gate_up, int M, int I, int ld, void* q, float* scale, w8_stream_t stream)
{
    if (!gate_up || !q || !scale || M <= 0 || I <= 0 || ld < 2 * I) return W8_ERR_INVALID_ARG;
    if (I % 8 != 0 || ld % 8 != 0 || !aligned(gate_up, 16) || !aligned(q, 8) || !aligned(scale, 4))
        return W8_ERR_ALIGNMENT;
    if (I > kRowMaxK) return W8_ERR_UNSUPPORTED;
    int rc = check_device(nullptr);
    if (rc != W8_OK) return rc;
    return launch_silu_mul_quant(gate_up, M, I, ld, q, scale, 0, 0, reinterpret_cast<cudaStream_t>(stream));
}

int w8_silu_mul_quant_group(const void* gate_up, int M, int I, int ld, int group, int ue8m0, void* q, float* scale,
                            w8_stream_t stream)
{
    if (!gate_up || !q || !scale || M <= 0 || I <= 0 || ld < 2 * I) return W8_ERR_INVALID_ARG;
    if (group != 128 || I % group != 0) return W8_ERR_UNSUPPORTED;
    if (ld % 8 != 0 || !aligned(gate_up, 16) || !aligned(q, 8) || !aligned(scale, 4)) return W8_ERR_ALIGNMENT;
    if (I > kRowMaxK) return W8_ERR_UNSUPPORTED;
    int rc = check_device(nullptr);
    if (rc != W8_OK) return rc;
    return launch_silu_mul_quant(gate_up, M, I, ld, q, scale, group, ue8m0, reinterpret_cast<cudaStream_t>(stream));
}

int w8_gemm(int fmt, const void* A_q, const float* A_scale, const void* W_q, const float* W_scale, void* out, int M,
            int N, int K, int variant, void* workspace, size_t ws_bytes, w8_stream_t stream)
{
    if (!out) return W8_ERR_INVALID_ARG;
    return gemm_common(fmt, A_q, A_scale, W_q, W_scale, out, nullptr, M, N, K, variant, workspace, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

int w8_gemm_i32_debug(const void* A_q, const void* W_q, int32_t* acc, int M, int N, int K, int variant,
                      void* workspace, size_t ws_bytes, w8_stream_t stream)
{
    if (!acc) return W8_ERR_INVALID_ARG;
    return gemm_common(W8_FMT_INT8, A_q, nullptr, W_q, nullptr, nullptr, acc, M, N, K, variant, workspace, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

int w8_gemm_timeout_debug(int fmt, const void* A_q, const float* A_scale, const void* W_q, const float* W_scale,
                          void* out, int M, int N, int K, int variant, int wait_us, w8_stream_t stream)
{
    if (!A_q || !W_q || !out || !A_scale || !W_scale) return W8_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0 || wait_us < 1 || wait_us > 1000000) return W8_ERR_INVALID_ARG;
    if (!aligned(A_q, 16) || !aligned(W_q, 16) || !aligned(out, 2)) return W8_ERR_ALIGNMENT;
    int sms = 0;
    int rc = check_device(&sms);
    if (rc != W8_OK) return rc;
    GemmPlan plan;
    rc = resolve(fmt, M, N, K, variant, sms, &plan);
    if (rc < 0) return rc;
    if (!plan.decode) return W8_ERR_UNSUPPORTED;
    return gemm_launch(plan, A_q, A_scale, W_q, W_scale, out, nullptr, nullptr, 0, reinterpret_cast<cudaStream_t>(stream),
                       nullptr, 1, (unsigned long long)wait_us * 1000ull);
}

int w8_gemm_resolve_variant(int fmt, int M, int N, int K, int variant)
{
    int sms = 0;
    if (check_device(&sms) != W8_OK) sms = 148;   // planning only: usable without a device
    GemmPlan plan;
    return resolve(fmt, M, N, K, variant, sms, &plan);
}

size_t w8_gemm_workspace_size(int fmt, int M, int N, int K, int variant)
{
    int sms = 0;
    if (check_device(&sms) != W8_OK) sms = 148;
    GemmPlan plan;
    if (resolve(fmt, M, N, K, variant, sms, &plan) < 0) return (size_t)-1;
    return plan.ws_bytes;
}

int w8_gemm_occupancy(int fmt, int M, int N, int K, int variant)
{
    int sms = 0;
    int rc = check_device(&sms);
    if (rc != W8_OK) return rc;
    GemmPlan plan;
    rc = resolve(fmt, M, N, K, variant, sms, &plan);
    if (rc < 0) return rc;
    int n = 0;
    rc = gemm_occupancy(plan, &n);
    return rc == W8_OK ? n : rc;
}

int w8_linear(int fmt, const void* x, int ldx, const void* W_q, const float* W_scale, void* out, int M, int N, int K,
              int variant, void* workspace, size_t ws_bytes, w8_stream_t stream)
{
    return linear_common(fmt, x, ldx, W_q, W_scale, out, M, N, K, variant, workspace, ws_bytes, nullptr, nullptr,
                         reinterpret_cast<cudaStream_t>(stream));
}

int w8_linear_debug(int fmt, const void* x, int ldx, const void* W_q, const float* W_scale, void* out, int M, int N,
                    int K, int variant, void* workspace, size_t ws_bytes, void* q_out, float* s_out, w8_stream_t stream)
{
    if (!q_out || !s_out) return W8_ERR_INVALID_ARG;
    return linear_common(fmt, x, ldx, W_q, W_scale, out, M, N, K, variant, workspace, ws_bytes,
                         static_cast<uint8_t*>(q_out), s_out, reinterpret_cast<cudaStream_t>(stream));
}

int w8_linear_resolve(int fmt, int M, int N, int K, int variant)
{
    int sms = 0;
    if (check_device(&sms) != W8_OK) sms = 148;
    GemmPlan plan;
    const int v = resolve(fmt, M, N, K, variant, sms, &plan);
    if (v < 0 || !(v & W8_V_FUSED)) return v;
    const int rc = linear_plan(fmt, M, N, K, v & ~W8_V_FUSED, sms, &plan);
    return rc == W8_OK ? v : rc;
}

size_t w8_linear_workspace_size(int fmt, int M, int N, int K, int variant)
{
    int sms = 0;
    if (check_device(&sms) != W8_OK) sms = 148;
    GemmPlan plan;
    if (resolve(fmt, M, N, K, variant, sms, &plan) < 0) return (size_t)-1;
    return linear_ws(plan);
}

int w8_load_table(const char* path)
{
    if (!path) return W8_ERR_INVALID_ARG;
    FILE* f = std::fopen(path, "r");
    if (!f) return W8_ERR_IO;
    std::vector<Entry> t;
    char line[512];
    bool bad = false;
    while (std::fgets(line, sizeof line, f)) {
        char* hash = std::strchr(line, '#');
        if (hash) *hash = 0;
        Entry e;
        unsigned v = 0;
        char extra[4];
        int n = std::sscanf(line, "%d %d %d %d %x %3s", &e.fmt, &e.N, &e.K, &e.m_max, &v, extra);
        if (n <= 0) continue;   // blank or comment
        if (n != 5 || e.fmt < 0 || e.fmt > 3 || e.N <= 0 || e.K <= 0 || e.m_max <= 0 || !(v & W8_V_EXPLICIT)) {
            bad = true;
            break;
        }
        e.variant = (int)v;
        t.push_back(e);
    }
    std::fclose(f);
    if (bad) return W8_ERR_IO;
    std::lock_guard<std::mutex> lk(g_tab_mu);
    g_table.swap(t);
    return (int)g_table.size();
}

void w8_clear_table(void)
{
    std::lock_guard<std::mutex> lk(g_tab_mu);
    g_table.clear();
}

int w8_device_status(int clear)
{
    const int g = gemm_device_status(clear);
    const int q = qknr_device_status(clear);
    if (g == W8_ERR_CUDA || q == W8_ERR_CUDA) return W8_ERR_CUDA;
    return g != 0 ? g : q;
}

int w8_grouped_gemm(int fmt, const void* A_q, const float* A_scale, const void* W_q, const float* W_scale, void* out,
                    const int* expert_offsets, int E, int T, int N, int K, int max_tokens_per_expert, int variant,
                    void* workspace, size_t ws_bytes, w8_stream_t stream)
{
    if (!A_q || !A_scale || !W_q || !W_scale || !out || !expert_offsets) return W8_ERR_INVALID_ARG;
    if (E <= 0 || T <= 0 || N <= 0 || K <= 0 || max_tokens_per_expert <= 0) return W8_ERR_INVALID_ARG;
    if (!aligned(A_q, 16) || !aligned(W_q, 16) || !aligned(out, 2) || !aligned(expert_offsets, 4)) return W8_ERR_ALIGNMENT;
    int sms = 0;
    int rc = check_device(&sms);
    if (rc != W8_OK) return rc;
    const int mm = max_tokens_per_expert < T ? max_tokens_per_expert : T;
    const int v = (variant & W8_V_EXPLICIT) ? variant : (grouped_variant(mm) | (variant & W8_V_PDL));
    GemmPlan plan;
    rc = grouped_plan(fmt, T, N, K, E, mm, v, sms, &plan);
    if (rc != W8_OK) return rc;
    return gemm_launch(plan, A_q, A_scale, W_q, W_scale, out, nullptr, workspace, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream), expert_offsets);
}

size_t w8_grouped_gemm_workspace_size(int fmt, int E, int T, int N, int K, int max_tokens_per_expert, int variant)
{
    int sms = 0;
    if (check_device(&sms) != W8_OK) sms = 148;
    if (T <= 0 || max_tokens_per_expert <= 0) return (size_t)-1;
    const int mm = max_tokens_per_expert < T ? max_tokens_per_expert : T;
    const int v = (variant & W8_V_EXPLICIT) ? variant : (grouped_variant(mm) | (variant & W8_V_PDL));
    GemmPlan plan;
    if (grouped_plan(fmt, T, N, K, E, mm, v, sms, &plan) != W8_OK) return (size_t)-1;
    return plan.ws_bytes;
}

int w8_qk_norm_rope(const void* qkv, void* out, int T, int Hq, int Hkv, int D, const void* q_weight,
                    const void* k_weight, const float* cos_sin, int max_pos, const int64_t* positions, float eps,
                    w8_stream_t stream)
{
    if (!qkv || !out || !q_weight || !k_weight || !cos_sin || !positions) return W8_ERR_INVALID_ARG;
    if (T < 0 || Hq < 0 || Hkv < 0 || max_pos <= 0 || !(eps >= 0.0f)) return W8_ERR_INVALID_ARG;
    if (D != 64 && D != 128 && D != 256) return W8_ERR_UNSUPPORTED;
    if (!aligned(qkv, 16) || !aligned(out, 16) || !aligned(q_weight, 16) || !aligned(k_weight, 16) ||
        !aligned(cos_sin, 16) || !aligned(positions, 8))
        return W8_ERR_ALIGNMENT;
    int rc = check_device(nullptr);
    if (rc != W8_OK) return rc;
    return launch_qk_norm_rope(qkv, out, T, Hq, Hkv, D, q_weight, k_weight, cos_sin, max_pos,
                               reinterpret_cast<const long long*>(positions), eps, reinterpret_cast<cudaStream_t>(stream));
}

const char* w8_status_string(int status)
{
    switch (status) {
    case W8_OK: return "ok";
    case W8_ERR_INVALID_ARG: return "invalid argument";
    case W8_ERR_UNSUPPORTED: return "unsupported format, variant or size";
    case W8_ERR_ALIGNMENT: return "misaligned pointer, stride or size";
    case W8_ERR_WORKSPACE: return "workspace missing or too small";
    case W8_ERR_CUDA: return "CUDA runtime error";
    case W8_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case W8_ERR_NO_DEVICE: return "current device is not an sm_100 GPU";
    case W8_ERR_IO: return "table file missing or malformed";
    default: return "unknown status";
    }
}

int w8_version(void) { return 1; }

}  // extern "C"
