// w8_internal.h -- declarations shared by the library's translation units (not part of
// the public ABI, which is include/w8.h).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/w8.h"

namespace w8 {

// ---- device / launch helpers (w8_api.cu) -------------------------------------------
int check_device(int* sm_count);   // W8_OK if the current device is sm_100; fills SM count

// ---- quantizers (w8_quant.cu) --------------------------------------------------------
int launch_quant_rows(int qfmt, const void* x, int M, int K, int ldx, void* q, float* scale, cudaStream_t s);
int launch_quant_group128(const void* x, int M, int K, int ldx, void* q, float* scale, int ue8m0, cudaStream_t s);
int launch_quant_weight_block(const void* w, int N, int K, void* q, float* scale, int ue8m0, cudaStream_t s);
int launch_rmsnorm_quant(const void* x, const void* gamma, float eps, int M, int H, int ldx, void* q, float* scale,
                         int group, int ue8m0, cudaStream_t s);
int launch_silu_mul_quant(const void* xgu, int M, int I, int ld, void* q, float* scale, int group, int ue8m0,
                          cudaStream_t s);

constexpr int kRowMaxK = 32768;   // longest row the register-resident row kernels accept

// ---- GEMM (w8_gemm.cu) -------------------------------------------------------------------
enum : int { kTileBN16 = 0, kTileBN32, kTileBN64, kTileBN128, kTileBN256, kNumTiles };

// Split partitions keep one int32 ticket counter per output tile in the first
// kMaxCounterTiles * 4 bytes of the workspace (256 KiB, the same for every shape).
constexpr int kMaxCounterTiles = 65536;

struct GemmPlan {
    int fmt;          // W8_FMT_*
    int M, N, K;
    int swap;         // 1: Swap-AB (MMA M slot over N)
    int bn;           // narrow tile side (16..256)
    int split;        // split_k (power of two) when !stream
    int stream;       // balanced partition over the SMs
    int stages;
    int pdl;
    int kps;          // 128-column K blocks per pipeline stage (1 or 2)
    int cluster;      // split_k chunks run as one thread-block cluster per tile
    int bm;           // rows of the MMA's M operand (128, or 64 for the narrow token tile)
    int pfix;         // split tiles finished by all their contributors, a column slice each
    int fq;           // the kernel quantizes the activations itself (w8_linear)
    int rg_max_kb;    // fq: K blocks of the largest activation region
    int fq_m8;        // fq: token rows staged from x (M rounded up to 8)
    int fq_xkb;       // fq: K blocks of x staged per CTA
    int fq_full_rows; // fq: whole rows staged (per-token maxima without a cluster split)
    int grouped;      // mixture-of-experts form: M = all tokens, N per expert
    int g_E;          // grouped: experts
    int pair;         // 256 x 256 tiles on CTA pairs (cta_group::2 MMA), Standard form
    int decode;       // decode form: tokens in the 64-row MMA operand, bn weight rows, split = cluster size
    int m8;           // decode: token rows of the activation box (M rounded up to 8)
    int l2ahead;      // decode: K blocks of weights kept in flight into L2 ahead of the stages
    int sw;           // decode: columns of the tile each cluster rank finishes (multiple of 16)
    int recv_R;       // decode: stages spanned by a rank's receive area
    int nkb_lo;       // decode: the smaller of the two K-block counts a rank holds
    int recv_first[2];   // decode: first stage of the receive area for nkb_lo and nkb_lo + 1 K blocks
    size_t a_region;  // decode with fq: bytes of the token-code region ahead of the stages
    // derived
    int rows_R, rows_C, r_tiles, c_tiles, tiles, kbs;
    int nsb;          // stage blocks (partition units) per tile
    long long units;
    int G;
    int align_tiles;
    size_t ws_counters;   // bytes of the counter area (0 if no partials)
    size_t ws_bytes;      // total workspace bytes
    size_t smem_bytes;
};

int gemm_plan(int fmt, int M, int N, int K, int variant, int sm_count, GemmPlan* p);
// starve / wait_ns (decode form only): the failure-path check of w8_gemm_timeout_debug
int gemm_launch(const GemmPlan& p, const void* A_q, const float* A_scale, const void* W_q, const float* W_scale,
                void* out, int32_t* out_i32, void* workspace, size_t ws_bytes, cudaStream_t s,
                const int* g_off = nullptr, int starve = 0, unsigned long long wait_ns = 0);
int gemm_occupancy(const GemmPlan& p, int* n);
int launch_qk_norm_rope(const void* qkv, void* out, int T, int Hq, int Hkv, int D, const void* q_weight,
                        const void* k_weight, const float* cos_sin, int max_pos, const long long* positions, float eps,
                        cudaStream_t s);
int qknr_device_status(int clear);
// plan of the fused quantize + GEMM form of `variant`: Swap-AB with every token in one
// narrow tile; W8_ERR_UNSUPPORTED when the variant has no such form
int linear_plan(int fmt, int M, int N, int K, int variant, int sm_count, GemmPlan* p);
// plan of the grouped (mixture-of-experts) GEMM: T tokens sorted by expert, E experts of
// N x K weights, at most max_m tokens per expert (sizes the token tiles and counters)
int grouped_plan(int fmt, int T, int N, int K, int E, int max_m, int variant, int sm_count, GemmPlan* p);
// fused launch: x bf16 [M, K] (row stride ldx) is quantized inside the GEMM kernel;
// dbg_q / dbg_s (optional) receive the codes and scales of weight tile 0's K blocks
int linear_launch(const GemmPlan& p, const void* x, int ldx, const void* W_q, const float* W_scale, void* out,
                  void* workspace, size_t ws_bytes, uint8_t* dbg_q, float* dbg_s, cudaStream_t s);
int gemm_device_status(int clear);

// ---- per-shape variant table (w8_api.cu) ---------------------------------------------
int table_lookup(int fmt, int N, int K, int M);   // explicit variant or 0 when absent

}  // namespace w8
