// w8_gemm_kernel.cuh -- the scaled 8-bit GEMM kernel template: one sm_100a kernel family (tcgen05 MMA, TMEM
// accumulators, TMA shared-memory pipeline) whose Standard, Split-K and Swap-AB forms
// are run-time choices, for FP8-dynamic, W8A8-INT8 and Block-FP8.
//
// What it computes ("Helion DSL added to vLLM to autotune linear inference backends",
// section "Unified GEMM Architecture"; "Helion nel backend vLLM: un solo GEMM ...",
// paragraphs 2-3; "PyTorch integra Helion en vLLM para acelerar inferencia FP8",
// section "Kernels Helion implementados": scaled_mm, scaled_mm_blockwise):
//   FP8_DYN  out[m,n] = bf16( sum_k A[m,k] W[n,k] * sA[m] * sW[n] ), fp32 accumulation
//   INT8     out[m,n] = bf16( float(sum_k A W as int32) * sA[m] * sW[n] )
//   BLOCK    out[m,n] = bf16( sum_kb sA[m,kb] sW[n/128,kb] sum_{k in kb} A W )
//
// Structure.  Both operands are K-major byte matrices.  The MMA's 128-row operand "R"
// and its BN-row operand "C" are bound at launch: Standard binds R = A (tokens) and
// C = W; Swap-AB binds R = W and C = A, so the accumulator is out^T and the epilogue
// writes the transpose (the pages' A@B = (B^T A^T)^T).  The problem is cut into units
// (output tile, 128-column K block).  CTA g owns the contiguous unit range
// [g*U/G, (g+1)*U/G): with G = tiles * split_k each CTA holds one 1/split_k K-chunk of
// one tile (Split-K); with G = the SM count the units are dealt out evenly (a
// balanced split); with whole-tile ranges nothing is split (Standard).  A tile whose K
// range is shared by several CTAs is finished by whichever arrives last (an atomic
// ticket, no waiting): it adds the fp32 (int32 for INT8) partials of the contributors
// in CTA order, which fixes the summation order, applies the scales and stores bf16.
//
// Per CTA (192 threads): warp 0 = TMA producer, warp 1 = TMEM allocator + MMA issuer
// (one elected lane), warps 2..5 = epilogue (TMEM -> registers -> scales -> global).
// Shared memory holds `stages` (R, C) tile pairs, 128-byte swizzled, behind full/empty
// mbarriers; the accumulator is double-buffered in TMEM (tfull/tempty mbarriers) so
// the epilogue of one tile overlaps the MMAs of the next.  Block-FP8 hands each
// 128-column K block to the epilogue, which scales it and accumulates in fp32
// registers.  Every wait is bounded by the global timer; on expiry the CTA records
// W8_ERR_DEVICE_TIMEOUT in the device status word, unwinds and frees its TMEM.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "w8_codes.cuh"
#include "w8_internal.h"
#include "w8_ptx.cuh"

namespace w8 {
namespace gemm {

// first device-side error (0 = none); one word per translation unit that instantiates
// kernels, read through that unit's status accessor
static __device__ int g_device_status;


constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kEpiBarrier = 1;          // named barrier id of the epilogue warps
constexpr int kTmemBarrier = 2;         // named barrier id of warps 1..5 (TMEM hand-off)
constexpr int kNumAcc = 2;              // TMEM accumulator barrier slots (buffers in use: kAccBufs)
constexpr unsigned long long kWaitNs = 1000000000ull;   // 1 s bound on any single wait
constexpr int kL2Ahead = 6;             // units whose weights are prefetched to L2 before the PDL wait

enum { KIND_F8 = 0, KIND_I8 = 1 };

struct GemmArgs {
    int M, N, K;
    int swap;
    int rows_R, rows_C;
    int r_tiles, c_tiles, tiles;
    int kbs;   // 128-column K blocks
    int nsb;   // stage blocks (units) per tile = ceil(kbs / KPS)
    long long units;
    int G;
    int align_tiles;
    int stages;
    int pdl;
    int ld_sblk;   // K/128: row length of the block-scale matrices
    int vec_ok;    // Standard epilogue may use 16-byte stores (N % 8 == 0, out 16-byte aligned)
    int csplit;    // cluster split: the K chunks of a tile are the CTAs of one cluster (0 = off)
    int pfix;      // 64-row token tile: split tiles are finished by all their contributors
    const uint8_t* w_ptr;   // weight codes [N, K] (for the L2 prefetch under PDL)
    const float* sA;
    const float* sW;
    __nv_bfloat16* out;
    int32_t* out_i32;
    uint32_t* partials;   // [G][2][BN][128] raw fp32 / int32 words
    int* counters;        // [tiles]
    // fused activation quantization (Swap-AB, every token in one C tile): the CTA reads
    // x bf16 [M, K] (row stride ldx) and writes the codes of the K blocks it needs into
    // shared memory itself
    const __nv_bfloat16* x;
    int ldx;
    int fq_block;         // 1: one scale per 1 x 128 group (Block-FP8); 0: per token
    int fq_ue8m0;         // group scales as powers of two
    int rg_max_kb;        // K blocks of the largest activation region over the CTAs
    int fq_m8;            // token rows staged from x (M rounded up to 8; rows past M are zero)
    int fq_xkb;           // K blocks of x staged per CTA (capacity)
    int fq_full_rows;     // stage whole rows (per-token maxima without a cluster split), else the region
    // grouped (mixture-of-experts) form: tokens sorted by expert, rows [g_off[e],
    // g_off[e+1]) of A belong to expert e, whose weights are rows [e N, (e+1) N) of W
    int grouped;
    int g_E;
    const int* g_off;     // device [g_E + 1]
    uint8_t* dbg_q;       // optional: codes of the K blocks of weight tile 0, [M, K]
    float* dbg_s;         // optional: scales, [M] or [M, K/128]
    // decode form (w8_gemm_decode.cu)
    int bn;               // weight rows per tile (64..256, a multiple of 16)
    int m8;               // token rows of the activation box
    int l2ahead;          // K blocks of weights prefetched into L2 ahead of the stages
    int sw;               // columns of the tile each cluster rank finishes
    int recv_R;           // stages spanned by a rank's receive area
    int nkb_lo;           // the smaller of the two K-block counts a rank holds
    int recv_first[2];    // first stage of the receive area for nkb_lo and nkb_lo + 1 K blocks
    int a_region;         // with the quantization fused: bytes of the token-code region
    // failure-path check (w8_gemm_timeout_debug): the producer issues no loads and every
    // wait gives up after wait_ns (0: the normal bound)
    int starve;
    unsigned long long wait_ns;
};

// K blocks a CTA with units [u0, u1) multiplies: its own range when the units lie in one
// tile, else every K block (a range that crosses a tile boundary wraps around in K).
__host__ __device__ inline void region_of(long long u0, long long u1, int nsb, int kps, int kbs, int* lo, int* n)
{
    if (u1 <= u0) { *lo = 0; *n = 0; return; }
    if (u0 / nsb == (u1 - 1) / nsb) {
        const int a = (int)(u0 % nsb) * kps;
        int b = (int)((u1 - 1) % nsb + 1) * kps;
        if (b > kbs) b = kbs;
        *lo = a;
        *n = b - a;
    } else {
        *lo = 0;
        *n = kbs;
    }
}

// Shared-memory bytes of the fused-quantization form: the activation region (codes), the
// staged bf16 rows of x, the stages (weights only), the barriers, and the per-token /
// per-group scale arrays.
__host__ __device__ inline size_t fq_smem_bytes(int bn, int kps, int stages, int rg_kb, int m8, int x_kb)
{
    const size_t region = (size_t)rg_kb * bn * 128;
    const size_t xstage = (size_t)x_kb * m8 * 256;
    const size_t ctrl = (size_t)(2 * stages + 2 * 2 + 6) * 8 + 16;
    const size_t scal = (size_t)(4 * bn + 8 * bn + bn * rg_kb) * 4;
    return 1024 + region + xstage + (size_t)stages * kps * 128 * 128 + ctrl + scal;
}

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor (tcgen05): K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row core-matrix groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);   // bits 0-13: start address >> 4
    d |= (uint64_t)(16u >> 4) << 16;             // bits 16-29: leading byte offset (unused here)
    d |= (uint64_t)(1024u >> 4) << 32;           // bits 32-45: stride byte offset
    d |= (uint64_t)1 << 46;                      // bits 46-47: descriptor version 1
    d |= (uint64_t)2 << 61;                      // bits 61-63: 128-byte swizzle
    return d;
}

// Instruction descriptor: dense, D = f32 (e4m3 x e4m3) or s32 (s8 x s8), both operands
// K-major, M = BM (64 or 128), N = BN.
template <int KIND, int BM, int BN>
__device__ __forceinline__ constexpr uint32_t instr_desc()
{
    return (KIND == KIND_I8 ? (2u << 4) : (1u << 4))      // bits 4-5: D format
           | (KIND == KIND_I8 ? (1u << 7) : 0u)           // bits 7-9: A format (s8 / e4m3)
           | (KIND == KIND_I8 ? (1u << 10) : 0u)          // bits 10-12: B format
           | ((uint32_t)(BN >> 3) << 17)                  // bits 17-22: N / 8
           | ((uint32_t)(BM >> 4) << 24);                 // bits 24-28: M / 16
}

// ---------------------------------------------------------------- unit partition
// U = total units and G = CTAs sharing them (a.units and a.G, or counted on the device
// in the grouped form, where CTAs past the unit count get nothing)
__device__ __forceinline__ long long unit_begin(const GemmArgs& a, long long g, long long U, long long G)
{
    if (a.align_tiles) return (g * a.tiles / a.G) * a.nsb;
    return g * U / G;
}

__device__ __forceinline__ int cta_of_unit(const GemmArgs& a, long long u, long long U, long long G)
{
    return (int)(((u + 1) * G - 1) / U);
}

// ---------------------------------------------------------------- bounded waits
__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_device_status, 0, code); }

// Poll an mbarrier phase until it completes, the deadline passes, or another role of
// this CTA has given up (abort flag).  Returns false on give-up.
template <bool CLUSTER_SCOPE = false>
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             uint64_t limit_ns = kWaitNs)
{
    auto probe = [&] { return CLUSTER_SCOPE ? ptx::mbar_try_wait_cluster(bar, parity) : ptx::mbar_try_wait(bar, parity); };
    if (probe()) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (probe()) return true;
        if ((it & 255u) == 0) {
            if (*abort_flag) return false;
            if (ptx::globaltimer_ns() - t0 > limit_ns) {
                *abort_flag = 1;
                record_error(W8_ERR_DEVICE_TIMEOUT);
                return false;
            }
        }
    }
}

// Poll a global counter until it reaches `target` (acquire, GPU scope), bounded like
// wait_bounded.  Used by the parallel fixup, whose contributors are all resident.
__device__ __forceinline__ bool wait_count(const int* p, int target, volatile int* abort_flag)
{
    auto probe = [&] {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
        return v >= target;
    };
    if (probe()) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(64);
        if (probe()) return true;
        if ((it & 63u) == 0) {
            if (*abort_flag) return false;
            if (ptx::globaltimer_ns() - t0 > kWaitNs) {
                *abort_flag = 1;
                record_error(W8_ERR_DEVICE_TIMEOUT);
                return false;
            }
        }
    }
}

// ---------------------------------------------------------------- epilogue helpers
template <int KIND>
__device__ __forceinline__ float word_to_float(uint32_t w)
{
    return KIND == KIND_I8 ? (float)(int32_t)w : __uint_as_float(w);
}

template <int KIND>
__device__ __forceinline__ uint32_t add_words(uint32_t x, uint32_t y)
{
    return KIND == KIND_I8 ? (uint32_t)((int32_t)x + (int32_t)y) : __float_as_uint(__fadd_rn(__uint_as_float(x), __uint_as_float(y)));
}

// Store one output element (row i of the R tile, column j of the C tile).  `w` is the
// raw accumulator word: unscaled (FP8/INT8) or already block-scaled (BLOCK).
// Swap-AB: [m_lo, m_hi) bounds the output rows (tokens, the C side) a tile may write --
// its own tokens; in the grouped form the neighbouring rows belong to other experts
template <int KIND, bool BLOCK>
__device__ __forceinline__ void store_out(const GemmArgs& a, const float* tokscale, int r_row, int c_row, uint32_t w,
                                          float s_row, int m_lo = 0, int m_hi = 0x7FFFFFFF)
{
    const int m = a.swap ? c_row : r_row;
    const int n = a.swap ? r_row : c_row;
    if (m >= a.M || n >= a.N) return;
    if (a.swap && (m < m_lo || m >= m_hi)) return;
    const size_t o = (size_t)m * a.N + n;
    if (KIND == KIND_I8 && a.out_i32 != nullptr) {
        a.out_i32[o] = (int32_t)w;
        return;
    }
    float v = word_to_float<KIND>(w);
    if (!BLOCK) {
        // s_row is the scale of the R-side index; the C-side scale is looked up here (the
        // token scales are global, or shared when the kernel quantized the activations)
        const float s_col = a.swap ? tokscale[m] : __ldg(a.sW + n);
        v = a.swap ? __fmul_rn(__fmul_rn(v, s_col), s_row) : __fmul_rn(__fmul_rn(v, s_row), s_col);
    }
    a.out[o] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Store 16 consecutive C-tile columns [c_base, c_base + 16) of R-tile row r_row.  In the
// Standard form these are 16 consecutive outputs of one row: two 16-byte stores.
template <int KIND, bool BLOCK>
__device__ __forceinline__ void store_chunk16(const GemmArgs& a, const float* tokscale, int r_row, int c_base,
                                              const uint32_t (&v)[16], float s_row, int m_lo = 0, int m_hi = 0x7FFFFFFF)
{
    if (!a.swap && a.vec_ok && a.out_i32 == nullptr && r_row < a.M && c_base + 15 < a.N) {
        float f[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
            f[jj] = word_to_float<KIND>(v[jj]);
            if (!BLOCK) f[jj] = __fmul_rn(__fmul_rn(f[jj], s_row), __ldg(a.sW + c_base + jj));
        }
        uint4 lo, hi;
        lo.x = pack_bf16x2(f[0], f[1]);   lo.y = pack_bf16x2(f[2], f[3]);
        lo.z = pack_bf16x2(f[4], f[5]);   lo.w = pack_bf16x2(f[6], f[7]);
        hi.x = pack_bf16x2(f[8], f[9]);   hi.y = pack_bf16x2(f[10], f[11]);
        hi.z = pack_bf16x2(f[12], f[13]); hi.w = pack_bf16x2(f[14], f[15]);
        uint4* dst = reinterpret_cast<uint4*>(a.out + (size_t)r_row * a.N + c_base);
        dst[0] = lo;
        dst[1] = hi;
        return;
    }
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) store_out<KIND, BLOCK>(a, tokscale, r_row, c_base + jj, v[jj], s_row, m_lo, m_hi);
}

__device__ __forceinline__ bool first_epi_thread(unsigned t) { return t == 64; }

// ---------------------------------------------------------------- the kernel
// BM = rows of the MMA's M operand ("R": 128, or 64 for a narrow token tile), BN = rows
// of its N operand ("C"), KPS = 128-column K blocks per pipeline stage (1 or 2).  A
// "unit" of the partition is one stage block of KPS K blocks of one output tile.
// Accumulator row r of a BM = 64 MMA lives in TMEM lane (r % 16) + 32 * (r / 16); of a
// BM = 128 MMA in lane r.
template <int BM, int BN, int KIND, bool BLOCK, int KPS, bool FQ = false, bool GRP = false>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmC, const GemmArgs a)
{
    constexpr int kRBytes = BM * 128;
    constexpr int kCBytes = BN * 128;
    // with fused activation quantization the stages carry weights only; the activation
    // codes sit in a region of their own, written once by the epilogue warps
    constexpr int kStageBytes = KPS * (kRBytes + (FQ ? 0 : kCBytes));
    // accumulators in TMEM, double-buffered (2 x BN <= 512 columns)
    constexpr int kAccBufs = 2;
    constexpr uint32_t kTmemCols = (kAccBufs * BN <= 32) ? 32 : (kAccBufs * BN <= 64) ? 64 : (kAccBufs * BN <= 128) ? 128 : (kAccBufs * BN <= 256) ? 256 : 512;
    constexpr uint32_t kIdesc = instr_desc<KIND, BM, BN>();

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = a.stages;
    uint8_t* region = smem;   // FQ: activation codes [K block][BN rows x 128 B], 128-byte swizzled
    // FQ: bf16 rows of x as loaded by TMA, [K block][fq_m8 rows][128 elements]
    uint8_t* xstage = smem + (FQ ? (size_t)a.rg_max_kb * kCBytes : 0);
    uint8_t* sbase = xstage + (FQ ? (size_t)a.fq_xkb * a.fq_m8 * 256 : 0);
    uint64_t* full = reinterpret_cast<uint64_t*>(sbase + (size_t)S * kStageBytes);
    uint64_t* empty = full + S;
    uint64_t* tfull = empty + S;
    uint64_t* tempty = tfull + kNumAcc;
    uint64_t* drain = tempty + kNumAcc;
    uint64_t* red_full = drain + 1;   // cluster split (rank 0): partials of the other ranks have landed
    uint64_t* red_go = red_full + 1;  // cluster split (ranks 1..): rank 0's stage memory is free
    uint64_t* a_ready = red_go + 1;   // FQ: the activation region is written
    uint64_t* amax_full = a_ready + 1;   // FQ, cluster split: the other ranks' partial row maxima landed
    uint64_t* x_full = amax_full + 1;    // FQ: the staged rows of x landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(x_full + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* ticket = reinterpret_cast<volatile int*>(tmem_slot + 2);
    // FQ scale arrays: per token scale, divisor (s', 1/s', factor), partial maxima of every
    // cluster rank, and the group scales of the region
    float* s_tok = reinterpret_cast<float*>(tmem_slot + 4);
    float* s_div = s_tok + BN;                                   // [3][BN]
    uint32_t* amax_slots = reinterpret_cast<uint32_t*>(s_div + 3 * BN);   // [8][BN]
    float* s_blk = reinterpret_cast<float*>(amax_slots + 8 * BN);          // [BN][rg_max_kb]
    // cluster split: [csplit - 1][BN columns][BM rows] partial words, written into rank 0's
    // stage memory once its last MMA has completed (the stages are free by then)
    uint32_t* red_buf = reinterpret_cast<uint32_t*>(sbase);
    // stage s: R slots [KPS][128 x 128 B], then C slots [KPS][BN x 128 B]; all 1024-aligned
    auto r_slot = [&](int s, int j) { return sbase + (size_t)s * kStageBytes + (size_t)j * kRBytes; };
    auto c_slot = [&](int s, int j) { return sbase + (size_t)s * kStageBytes + (size_t)KPS * kRBytes + (size_t)j * kCBytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(ptx::smem_u32(full + s), 1);
            ptx::mbar_init(ptx::smem_u32(empty + s), 1);
        }
        for (int b = 0; b < kNumAcc; ++b) {
            ptx::mbar_init(ptx::smem_u32(tfull + b), 1);
            ptx::mbar_init(ptx::smem_u32(tempty + b), kEpiThreads / 32);
        }
        ptx::mbar_init(ptx::smem_u32(drain), 1);
        ptx::mbar_init(ptx::smem_u32(red_full), a.csplit > 1 ? (uint32_t)(a.csplit - 1) * kEpiThreads : 1u);
        ptx::mbar_init(ptx::smem_u32(red_go), 1);
        ptx::mbar_init(ptx::smem_u32(a_ready), 1);
        ptx::mbar_init(ptx::smem_u32(amax_full), a.csplit > 1 ? (uint32_t)(a.csplit - 1) * 32u : 1u);
        ptx::mbar_init(ptx::smem_u32(x_full), 1);
        *abort_flag = 0;
        ptx::fence_barrier_init();
    }
    if (threadIdx.x == 32) {
        ptx::prefetch_tmap(&tmR);
        ptx::prefetch_tmap(&tmC);
    }
    __syncthreads();
    // cluster split: rank 0's reduction barrier must be initialised before any other
    // rank can arrive on it
    if (a.csplit > 1) ptx::cluster_sync();
    // TMEM is allocated by warp 1 and handed to warps 1..5 through a named barrier, so
    // the producer can start streaming while the allocation still waits for columns a
    // CTA of the previous kernel holds
    uint32_t tmem = 0;
    if (warp != 0) {
        if (warp == 1) {
            ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
            // Dependent kernels are released only once this CTA holds its TMEM columns: a
            // CTA of a dependent on the same SM then never takes columns this one still
            // needs (it would hold them while waiting for this grid to finish).
            if (lane == 0) ptx::grid_dep_launch();
        }
        ptx::tc_fence_before();
        ptx::bar_sync(kTmemBarrier, kThreads - 32);
        ptx::tc_fence_after();
        tmem = *tmem_slot;
    }

    const int nsb = a.nsb;   // stage blocks per tile
    const int kbs = a.kbs;   // 128-column K blocks per tile
    // grouped form: per-expert tile counts from the expert offsets (written by the kernels
    // ahead, hence after the wait), as prefix sums in shared memory; every CTA derives the
    // same balanced partition of the units of the experts that have tokens
    int* s_gtile = reinterpret_cast<int*>(tmem_slot + 4);     // [g_E + 1] tile prefix
    int* s_goff = s_gtile + (GRP ? a.g_E + 1 : 0);             // [g_E + 1] clamped offsets
    long long U = a.units;
    if (GRP) {
        ptx::grid_dep_wait();
        if (warp == 0) {
            const int E = a.g_E, T = a.rows_C;
            const int per = (E + 31) / 32;
            const int e0 = lane * per, e1 = min(e0 + per, E);
            // offsets must rise within [0, T]; otherwise nothing is computed and the
            // device status records W8_ERR_INVALID_ARG
            bool bad = false;
            for (int e = e0; e < e1; ++e) {
                const int lo = a.g_off[e], hi = a.g_off[e + 1];
                bad |= lo < 0 || hi > T || hi < lo;
            }
            const bool any_bad = __any_sync(0xFFFFFFFFu, bad);
            int tiles = 0;
            for (int e = e0; e < e1; ++e) {
                const int lo = any_bad ? 0 : a.g_off[e], hi = any_bad ? 0 : a.g_off[e + 1];
                s_goff[e] = lo;
                if (e == E - 1) s_goff[E] = hi;
                tiles += a.r_tiles * ((hi - lo + BN - 1) / BN);
            }
            // exclusive scan of the lanes' tile counts
            int incl = tiles;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += v;
            }
            int run = incl - tiles;
            for (int e = e0; e < e1; ++e) {
                s_gtile[e] = run;
                const int lo = any_bad ? 0 : a.g_off[e], hi = any_bad ? 0 : a.g_off[e + 1];
                run += a.r_tiles * ((hi - lo + BN - 1) / BN);
            }
            if (lane == 31) s_gtile[E] = incl;
            if (any_bad && lane == 0) record_error(W8_ERR_INVALID_ARG);
        }
        __syncthreads();
        U = (long long)s_gtile[a.g_E] * nsb;
    }
    // every CTA of the partition must own at least one unit (a split tile is finished by
    // its contributors, consecutive CTAs): with fewer units than CTAs the rest idle
    const long long Gp = (GRP && U < a.G) ? U : a.G;
    const long long u0 = ((long long)blockIdx.x < Gp) ? unit_begin(a, blockIdx.x, U, Gp) : U;
    const long long u1 = ((long long)blockIdx.x < Gp) ? unit_begin(a, blockIdx.x + 1, U, Gp) : U;
    // tile t -> weight tile rt, token tile ct, the rows they start at in W and A, and the
    // number of valid rows on the C side (tokens of the expert, in the grouped form).
    // Grouped: the token box starts at c_off + ct * BN unless that would run it past the
    // last token row; then it starts earlier (at row T - BN, or 0) and the tile's tokens
    // sit c_shift columns into it.
    auto tile_loc = [&](int t, int& rt, int& ct, int& r_off, int& c_off, int& c_valid, int& c_shift) {
        c_shift = 0;
        if (!GRP) {
            rt = t / a.c_tiles;
            ct = t % a.c_tiles;
            r_off = 0;
            c_off = 0;
            c_valid = a.rows_C;
            return;
        }
        // the expert e with s_gtile[e] <= t < s_gtile[e + 1] (it has tiles)
        int lo = 0, hi = a.g_E;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_gtile[mid] <= t) lo = mid; else hi = mid;
        }
        const int m_e = s_goff[lo + 1] - s_goff[lo];
        const int ctiles = (m_e + BN - 1) / BN;
        const int lt = t - s_gtile[lo];
        rt = lt / ctiles;
        ct = lt % ctiles;
        r_off = lo * a.rows_R;
        const int start = s_goff[lo] + ct * BN;
        const int box = min(start, max(0, a.rows_C - BN));
        c_shift = start - box;
        c_off = box - ct * BN;    // so that c_off + ct * BN is the box's first row
        c_valid = min(m_e, ct * BN + (BN - c_shift));   // tokens of this tile end by column BN
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_w = ptx::policy_evict_first();   // weights: streamed once
            const uint64_t pol_a = ptx::policy_evict_last();    // activations: re-read by every CTA
            const uint64_t pol_R = a.swap ? pol_w : pol_a;
            const uint64_t pol_C = a.swap ? pol_a : pol_w;
            const long long n = u1 - u0;
            // load the R boxes (load_r) and/or C boxes of unit u into stage s
            auto issue = [&](int s, long long u, bool load_r, bool load_c, bool expect) {
                const int t = (int)(u / nsb), kb0 = (int)(u % nsb) * KPS;
                const int nkb = (kbs - kb0 < KPS) ? kbs - kb0 : KPS;
                int rt, ct, r_off, c_off, c_valid, c_shift;
                tile_loc(t, rt, ct, r_off, c_off, c_valid, c_shift);
                const uint32_t fb = ptx::smem_u32(full + s);
                if (expect) ptx::mbar_arrive_expect_tx(fb, (uint32_t)(nkb * (kRBytes + (FQ ? 0 : kCBytes))));
                for (int j = 0; j < nkb; ++j) {
                    if (load_r) ptx::tma_load_2d(ptx::smem_u32(r_slot(s, j)), &tmR, fb, (kb0 + j) * 128, r_off + rt * BM, pol_R);
                    if (load_c && !FQ) ptx::tma_load_2d(ptx::smem_u32(c_slot(s, j)), &tmC, fb, (kb0 + j) * 128, c_off + ct * BN, pol_C);
                }
            };
            // With programmatic dependent launch, before waiting for the kernels ahead of
            // this one, the producer requests the weight boxes of the first `pre` stages
            // (weights are never the output of work in flight; the epilogue warps prefetch
            // the next units' weights into L2); the activation boxes follow after the wait.
            const int pre = (a.pdl && !GRP) ? (int)(n < S ? n : S) : 0;
            for (int i = 0; i < pre; ++i) issue(i, u0 + i, a.swap != 0, a.swap == 0, true);
            ptx::grid_dep_wait();
            if (FQ) {
                // stage the rows of x this CTA quantizes: its region with a cluster split
                // (the ranks together cover K), else the whole rows (their maxima need it)
                int xlo = 0, xn = kbs;
                if (!a.fq_full_rows) region_of(u0, u1, nsb, KPS, kbs, &xlo, &xn);
                const uint32_t xb = ptx::smem_u32(x_full);
                ptx::mbar_arrive_expect_tx(xb, (uint32_t)(xn * a.fq_m8 * 256));
                for (int j = 0; j < xn; ++j)
                    ptx::tma_load_2d(ptx::smem_u32(xstage + (size_t)j * a.fq_m8 * 256), &tmC, xb, (xlo + j) * 128, 0,
                                     pol_a);
            } else {
                for (int i = 0; i < pre; ++i) issue(i, u0 + i, a.swap == 0, a.swap != 0, false);
            }
            long long issued = pre;
            int stage = pre % S;
            uint32_t phase = (pre == S) ? 1u : 0u;
            for (long long i = pre; i < n; ++i) {
                if (!wait_bounded(ptx::smem_u32(empty + stage), phase ^ 1u, abort_flag)) break;
                issue(stage, u0 + i, true, true, true);
                ++issued;
                if (++stage == S) { stage = 0; phase ^= 1u; }
            }
            if (*abort_flag) {
                // let the copies still in flight land before the CTA unwinds: the last
                // min(S, issued) stages (earlier ones were consumed), each bounded
                const long long lo = issued > S ? issued - S : 0;
                for (long long j = lo; j < issued; ++j) {
                    const uint32_t fb = ptx::smem_u32(full + (int)(j % S));
                    const uint32_t par = (uint32_t)((j / S) & 1);
                    const uint64_t t0 = ptx::globaltimer_ns();
                    while (!ptx::mbar_try_wait(fb, par) && ptx::globaltimer_ns() - t0 < 10000000ull) {}
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // (its bounded waits start only once the kernels ahead of this one are done)
        ptx::grid_dep_wait();
        int stage = 0, buf = 0;
        uint32_t phase = 0, bphase = 0;
        bool ok = true;
        int rg_lo = 0, rg_n = 0;
        if (FQ) {
            // the activation codes come from this CTA's epilogue warps
            region_of(u0, u1, nsb, KPS, kbs, &rg_lo, &rg_n);
            if (lane == 0) {
                ok = wait_bounded(ptx::smem_u32(a_ready), 0, abort_flag);
                ptx::tc_fence_after();
            }
            ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
        }
        for (long long u = u0; u < u1 && ok; ++u) {
            const int sb = (int)(u % nsb);
            const int kb0 = sb * KPS;
            const int nkb = (kbs - kb0 < KPS) ? kbs - kb0 : KPS;
            const bool seg_first = (u == u0 || sb == 0);
            const bool seg_last = (u == u1 - 1 || sb == nsb - 1);
            int nbuf_used = 0;
            if (lane == 0) {
                if (!BLOCK && seg_first) {
                    ok = wait_bounded(ptx::smem_u32(tempty + buf), bphase ^ 1u, abort_flag);
                    ptx::tc_fence_after();
                }
                if (ok) ok = wait_bounded(ptx::smem_u32(full + stage), phase, abort_flag);
                if (ok) {
                    ptx::tc_fence_after();
                    int b = buf;
                    uint32_t bp = bphase;
                    for (int j = 0; j < nkb && ok; ++j) {
                        if (BLOCK) {
                            // every K block gets its own accumulator, handed to the epilogue
                            ok = wait_bounded(ptx::smem_u32(tempty + b), bp ^ 1u, abort_flag);
                            ptx::tc_fence_after();
                            if (!ok) break;
                        }
                        const uint64_t dR = smem_desc(ptx::smem_u32(r_slot(stage, j)));
                        const uint64_t dC = FQ ? smem_desc(ptx::smem_u32(region + (size_t)(kb0 + j - rg_lo) * kCBytes))
                                               : smem_desc(ptx::smem_u32(c_slot(stage, j)));
                        const uint32_t d_tmem = tmem + (uint32_t)(b * BN);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            // advance 32 K-bytes inside the 128-byte swizzle row: +2 in 16-byte units
                            const uint32_t acc = BLOCK ? (k > 0 ? 1u : 0u) : ((seg_first && j == 0 && k == 0) ? 0u : 1u);
                            if (KIND == KIND_I8) ptx::mma_i8(d_tmem, dR + 2 * k, dC + 2 * k, kIdesc, acc);
                            else                 ptx::mma_f8f6f4(d_tmem, dR + 2 * k, dC + 2 * k, kIdesc, acc);
                        }
                        if (BLOCK) {
                            ptx::mma_commit(ptx::smem_u32(tfull + b));
                            if (++b == kAccBufs) { b = 0; bp ^= 1u; }
                            ++nbuf_used;
                        }
                    }
                    if (ok) {
                        ptx::mma_commit(ptx::smem_u32(empty + stage));
                        if (!BLOCK && seg_last) ptx::mma_commit(ptx::smem_u32(tfull + buf));
                    }
                }
            }
            ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
            nbuf_used = __shfl_sync(0xFFFFFFFFu, nbuf_used, 0);
            if (++stage == S) { stage = 0; phase ^= 1u; }
            if (BLOCK) {
                for (int j = 0; j < nbuf_used; ++j)
                    if (++buf == kAccBufs) { buf = 0; bphase ^= 1u; }
            } else if (seg_last) {
                if (++buf == kAccBufs) { buf = 0; bphase ^= 1u; }
            }
        }
        if (!ok && lane == 0) {
            // MMAs already issued must finish before TMEM is released (bounded)
            ptx::mma_commit(ptx::smem_u32(drain));
            const uint64_t t0 = ptx::globaltimer_ns();
            while (!ptx::mbar_try_wait(ptx::smem_u32(drain), 0) && ptx::globaltimer_ns() - t0 < 10000000ull) {}
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        if (a.pdl && !FQ && !GRP) {
            // Idle until the first accumulator is ready: prefetch into L2 the weight rows
            // of the kL2Ahead units that follow the producer's first stages, so that the
            // weight stream keeps HBM busy while the kernels ahead of this one finish.
            const long long p0 = u0 + S, p1 = (u1 < p0 + kL2Ahead) ? u1 : p0 + kL2Ahead;
            const int wrows = a.swap ? BM : BN;
            const int lines_per_row = KPS;                  // 128-byte lines per row per unit
            const long long total = (p1 > p0) ? (p1 - p0) * wrows * lines_per_row : 0;
            for (long long e = threadIdx.x - 64; e < total; e += kEpiThreads) {
                const long long u = p0 + e / (wrows * lines_per_row);
                const int rem = (int)(e % (wrows * lines_per_row));
                const int t = (int)(u / nsb), kb = (int)(u % nsb) * KPS + rem % lines_per_row;
                const int row = (a.swap ? (t / a.c_tiles) * BM : (t % a.c_tiles) * BN) + rem / lines_per_row;
                if (row < a.N && kb < kbs) ptx::prefetch_l2_evict_last(a.w_ptr + (size_t)row * a.K + (size_t)kb * 128);
            }
        }
        ptx::grid_dep_wait();
        // token scales: global, or (FQ) the ones this CTA computes below
        const float* tokscale = FQ ? s_tok : a.sA;
        int rg_lo = 0, rg_n = 0;
        bool fq_ok = true;
        if (FQ) {
            // ---- fused activation quantization: the producer stages the bf16 rows of x
            // by TMA; from them: row (or group) maxima, scales, then the codes of every K
            // block this CTA multiplies, written 128-byte swizzled into the region the MMA
            // reads in place of a TMA-loaded activation tile
            region_of(u0, u1, nsb, KPS, kbs, &rg_lo, &rg_n);
            const int te = threadIdx.x - 64;
            const int M = a.M, K = a.K, m8 = a.fq_m8;
            const bool part = a.csplit > 1;
            const uint32_t rank = part ? ptx::cluster_ctarank() : 0u;
            const int xlo = a.fq_full_rows ? 0 : rg_lo;   // K block held by the first staged block
            const int xn = a.fq_full_rows ? kbs : rg_n;
            // before x arrives: zero codes for the rows past M, zero this rank's maxima
            for (int it = te; it < (BN - M) * rg_n * 8; it += kEpiThreads) {
                const int c16 = it & 7, kbl = (it >> 3) % rg_n, m = M + (it >> 3) / rg_n;
                *reinterpret_cast<uint4*>(region + (size_t)kbl * kCBytes + (size_t)m * 128 + (size_t)((c16 ^ (m & 7)) << 4)) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            for (int m = te; m < BN; m += kEpiThreads) amax_slots[rank * BN + m] = 0u;
            auto xrow = [&](int kb_staged, int m) {
                return reinterpret_cast<const uint4*>(xstage + ((size_t)kb_staged * m8 + m) * 256);
            };
            fq_ok = wait_bounded(ptx::smem_u32(x_full), 0, abort_flag);
            if (ptx::bar_red_or(kEpiBarrier, kEpiThreads, !fq_ok)) fq_ok = false;
            if (fq_ok && !a.fq_block) {
                // per-token maxima over the staged K blocks: every epilogue thread takes
                // 16-byte chunks of every row, then a warp maximum and a shared atomic
                // (non-negative floats order like their bit patterns)
                for (int m = 0; m < M; ++m) {
                    float mx = 0.0f;
                    for (int c = te; c < xn * 16; c += kEpiThreads) {
                        float f[8];
                        unpack_bf16x8(xrow(c >> 4, m)[c & 15], f);
#pragma unroll
                        for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(f[i]));
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
                    if (lane == 0 && mx > 0.0f) atomicMax(amax_slots + rank * BN + m, __float_as_uint(mx));
                }
                ptx::bar_sync(kEpiBarrier, kEpiThreads);
                if (part) {
                    // one warp per rank sends the partial maxima to the other ranks
                    // (distributed shared memory) and arrives on their barriers
                    if (te < 32) {
                        for (int m = te; m < M; m += 32)
                            for (int r = 0; r < a.csplit; ++r)
                                if ((uint32_t)r != rank)
                                    ptx::st_cluster_u32(ptx::map_to_rank(ptx::smem_u32(amax_slots + rank * BN + m), (uint32_t)r),
                                                        amax_slots[rank * BN + m]);
                        for (int r = 0; r < a.csplit; ++r)
                            if ((uint32_t)r != rank) ptx::mbar_arrive_remote(ptx::map_to_rank(ptx::smem_u32(amax_full), (uint32_t)r));
                    }
                    const bool w = wait_bounded<true>(ptx::smem_u32(amax_full), 0, abort_flag);
                    if (ptx::bar_red_or(kEpiBarrier, kEpiThreads, !w)) fq_ok = false;
                }
                if (fq_ok) {
                    const int nslots = part ? a.csplit : 1;
                    for (int m = te; m < m8; m += kEpiThreads) {
                        float amax = 0.0f;
                        if (m < M)
                            for (int r = 0; r < nslots; ++r) amax = fmaxf(amax, __uint_as_float(amax_slots[r * BN + m]));
                        const float s = scale_from_amax(amax, KIND == KIND_I8 ? kInt8Max : kE4M3Max, false);
                        const RowDivisor d = make_divisor(s);
                        s_tok[m] = s;
                        s_div[m] = d.s;
                        s_div[BN + m] = d.y;
                        s_div[2 * BN + m] = d.f;
                        if (a.dbg_s != nullptr && blockIdx.x == 0 && m < M) a.dbg_s[m] = s;
                    }
                    for (int m = m8 + te; m < BN; m += kEpiThreads) s_tok[m] = 1.0f;
                    ptx::bar_sync(kEpiBarrier, kEpiThreads);
                }
            }
            if (fq_ok) {
                // K blocks of weight tile 0 that this CTA multiplies (for the optional copy
                // of the codes)
                const int dbg_lo = (u0 < nsb) ? (int)u0 * KPS : kbs;
                const int dbg_hi = (u0 < nsb) ? (int)min(u1, (long long)nsb) * KPS : kbs;
                // items: (token row, K block, 16-code chunk); the 8 chunks of one row's K
                // block are 8 consecutive lanes, so a group's lanes are active together
                const int total = M * rg_n * 8;
                for (int it = te; it < total; it += kEpiThreads) {
                    const int c16 = it & 7;
                    const int kbl = (it >> 3) % rg_n;
                    const int m = (it >> 3) / rg_n;
                    const int kb = rg_lo + kbl;
                    const int k0 = kb * 128 + c16 * 16;
                    float f[16];
                    {
                        const uint4* src = xrow(kb - xlo, m) + 2 * c16;
                        float lo[8], hi[8];
                        unpack_bf16x8(src[0], lo);
                        unpack_bf16x8(src[1], hi);
#pragma unroll
                        for (int i = 0; i < 8; ++i) { f[i] = lo[i]; f[8 + i] = hi[i]; }
                    }
                    RowDivisor d;
                    if (a.fq_block) {
                        // one scale per 1 x 128 group: the maximum over the group's 8 lanes
                        const unsigned gmask = 0xFFu << (lane & 24);
                        float mx = 0.0f;
#pragma unroll
                        for (int i = 0; i < 16; ++i) mx = fmaxf(mx, fabsf(f[i]));
#pragma unroll
                        for (int o = 1; o < 8; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(gmask, mx, o));
                        const float s = scale_from_amax(mx, kE4M3Max, a.fq_ue8m0 != 0);
                        d = make_divisor(s);
                        if (c16 == 0) s_blk[m * a.rg_max_kb + kbl] = s;
                        if (c16 == 0 && a.dbg_s != nullptr && kb >= dbg_lo && kb < dbg_hi) a.dbg_s[(size_t)m * kbs + kb] = s;
                    } else {
                        d.s = s_div[m];
                        d.y = s_div[BN + m];
                        d.f = s_div[2 * BN + m];
                    }
                    uint32_t w4[4];
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const float q0 = quotient_rn(f[4 * g], d), q1 = quotient_rn(f[4 * g + 1], d);
                        const float q2 = quotient_rn(f[4 * g + 2], d), q3 = quotient_rn(f[4 * g + 3], d);
                        w4[g] = (KIND == KIND_I8)
                                    ? (int8_code(q0) | (int8_code(q1) << 8) | (int8_code(q2) << 16) | (int8_code(q3) << 24))
                                    : (e4m3x2(q0, q1) | (e4m3x2(q2, q3) << 16));
                    }
                    const uint4 codes = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    *reinterpret_cast<uint4*>(region + (size_t)kbl * kCBytes + (size_t)m * 128 + (size_t)((c16 ^ (m & 7)) << 4)) =
                        codes;
                    if (a.dbg_q != nullptr && k0 < K && kb >= dbg_lo && kb < dbg_hi)
                        *reinterpret_cast<uint4*>(a.dbg_q + (size_t)m * K + k0) = codes;
                }
                // the tensor core reads the region through the async proxy
                ptx::fence_proxy_async_smem();
                ptx::bar_sync(kEpiBarrier, kEpiThreads);
                if (first_epi_thread(threadIdx.x)) ptx::mbar_arrive(ptx::smem_u32(a_ready));
            }
        }
        const int q = warp & 3;                 // TMEM lane quadrant of this warp
        // row of the R tile held by this thread (BM = 64: lanes 16..31 of a quadrant hold none)
        const int i = (BM == 128) ? q * 32 + lane : q * 16 + (lane & 15);
        const bool lane_has_row = (BM == 128) || lane < 16;
        const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
        const bool first_epi = (threadIdx.x == 64);
        constexpr int kAccRegs = BLOCK ? BN : 1;
        // parallel fixup (64-row token tile): split tiles this CTA contributed to, finished
        // after its last segment (at most its first and its last segment are split)
        int fix_t[2] = {0, 0};
        int nfix = 0;
        int buf = 0;
        uint32_t bphase = 0;
        bool ok = fq_ok;
        for (long long u = u0; u < u1 && ok;) {
            const int t = (int)(u / nsb);
            const int sb_lo = (int)(u % nsb);
            const long long rem = u1 - u;
            const int sb_hi = (int)((nsb - sb_lo < rem) ? nsb : sb_lo + rem);
            int rt, ct, r_off, c_off, c_valid, c_shift;
            tile_loc(t, rt, ct, r_off, c_off, c_valid, c_shift);
            // sentinel for threads holding no real row: padding lanes of the 64-row tile and,
            // in the Standard form, token rows past M (their accumulators are zero)
            const int r_row = (lane_has_row && rt * BM + i < a.rows_R) ? rt * BM + i : 0x7FFFFFFF;
            const bool has_row = r_row != 0x7FFFFFFF;
            const bool full_tile = (sb_lo == 0 && sb_hi == nsb);
            const int slot = (u == u0) ? 0 : 1;
            // scale of this thread's R-side index (FP8 / INT8; BLOCK scales per K block)
            float s_row = 1.0f;
            if (!BLOCK && a.out_i32 == nullptr && r_row < a.rows_R) s_row = __ldg((a.swap ? a.sW : a.sA) + r_off + r_row);

            float acc[kAccRegs];
#pragma unroll
            for (int j = 0; j < kAccRegs; ++j) acc[j] = 0.0f;
            if (BLOCK) {
                // ---- per-K-block promotion: acc += (sA * sW) * (block dot product), fp32
                const int kb_end = (sb_hi * KPS < kbs) ? sb_hi * KPS : kbs;
                for (int kb = sb_lo * KPS; kb < kb_end; ++kb) {
                    const bool w = wait_bounded(ptx::smem_u32(tfull + buf), bphase, abort_flag);
                    if (ptx::bar_red_or(kEpiBarrier, kEpiThreads, !w)) { ok = false; break; }
                    ptx::tc_fence_after();
                    // scales of this K block: swap -> sW scalar, sA per column (lane-loaded,
                    // shuffled); standard -> one product per thread
                    float sa_l[(BN + 31) / 32];
                    float sc_thread = 0.0f, sw = 0.0f;
                    if (a.swap) {
                        sw = __ldg(a.sW + (size_t)rt * a.ld_sblk + kb);
#pragma unroll
                        for (int h = 0; h < (BN + 31) / 32; ++h) {
                            const int jc = h * 32 + lane;
                            const int col = ct * BN + jc;
                            sa_l[h] = (jc < BN && col < a.rows_C)
                                          ? (FQ ? s_blk[col * a.rg_max_kb + (kb - rg_lo)] : __ldg(a.sA + (size_t)col * a.ld_sblk + kb))
                                          : 0.0f;
                        }
                    } else {
                        const float sa = (r_row < a.rows_R) ? __ldg(a.sA + (size_t)r_row * a.ld_sblk + kb) : 0.0f;
                        sc_thread = __fmul_rn(sa, __ldg(a.sW + (size_t)((ct * BN) / 128) * a.ld_sblk + kb));
                    }
#pragma unroll
                    for (int c0 = 0; c0 < BN; c0 += 16) {
                        uint32_t v[16];
                        ptx::tmem_ld16(t_lane + (uint32_t)(buf * BN + c0), v);
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) {
                            const int j = c0 + jj;
                            const float sc = a.swap ? __fmul_rn(__shfl_sync(0xFFFFFFFFu, sa_l[j / 32], j % 32), sw)
                                                    : sc_thread;
                            acc[BLOCK ? j : 0] = __fmaf_rn(__uint_as_float(v[jj]), sc, acc[BLOCK ? j : 0]);
                        }
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(tempty + buf));
                    if (++buf == kAccBufs) { buf = 0; bphase ^= 1u; }
                }
                if (!ok) break;
            } else {
                const bool w = wait_bounded(ptx::smem_u32(tfull + buf), bphase, abort_flag);
                if (ptx::bar_red_or(kEpiBarrier, kEpiThreads, !w)) { ok = false; break; }
                ptx::tc_fence_after();
            }

            // 16 accumulator words of column chunk c0: from TMEM (FP8/INT8) or registers (BLOCK)
            auto fetch16 = [&](int c0, uint32_t (&v)[16]) {
                if (BLOCK) {
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) v[jj] = __float_as_uint(acc[BLOCK ? (c0 + jj) % kAccRegs : 0]);
                } else {
                    ptx::tmem_ld16(t_lane + (uint32_t)(buf * BN + c0), v);
                }
            };

            // columns of this tile that hold real rows of the C operand (tokens for
            // Swap-AB: only these are written, published and reduced)
            // columns [c_shift, ncv) of the tile are its tokens (c_shift > 0 only in the
            // grouped form, where the box may start before the tile's first token)
            const int ncv = c_shift + ((c_valid - ct * BN < BN - c_shift) ? c_valid - ct * BN : BN - c_shift);
            const int c_base = c_off + ct * BN;   // first output row (Swap-AB) / column of this tile
            const int m_lo = c_base + c_shift;    // first token this tile may write
            const int m_hi = c_base + ncv;        // one past its last
            // 64-row token tile: only nrows rows are real tokens; its partials are kept as
            // [row][column] and reduced column-parallel by all 128 epilogue threads
            constexpr bool kCompact = (BM == 64);
            const int nrows = (a.rows_R - rt * BM < BM) ? a.rows_R - rt * BM : BM;
            const int te = threadIdx.x - 64;   // epilogue thread index 0..127
            // publish this thread's row (if any) as BN contiguous words at dst (generic or
            // cluster-shared address space)
            auto publish_row = [&](uint32_t* gdst, uint32_t sdst, bool remote) {
#pragma unroll
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    if (c0 >= ncv) break;
                    uint32_t v[16];
                    fetch16(c0, v);
                    if (has_row) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            if (remote) {
                                ptx::st_cluster_v4(sdst + (uint32_t)((c0 + 4 * q4) * 4), v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
                            } else {
                                uint4 w4 = make_uint4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
                                __stcg(reinterpret_cast<uint4*>(gdst + c0 + 4 * q4), w4);
                            }
                        }
                    }
                }
            };
            // finish output column `col` of row r from a summed word
            auto finish = [&](int r, int col, uint32_t w) {
                const int m = rt * BM + r;
                const float sr = (a.out_i32 == nullptr) ? __ldg(a.sA + m) : 1.0f;
                store_out<KIND, BLOCK>(a, tokscale, m, ct * BN + col, w, sr);
            };
            if (kCompact && a.csplit > 1) {
                // ---- cluster split, 64-row token tile: every rank's real rows go to rank 0's
                // stage memory as [rank][row][column]; rank 0 sums ranks in order per column
                const uint32_t rank = ptx::cluster_ctarank();
                const uint32_t slot_words = (uint32_t)(nrows * BN);
                if (rank != 0) {
                    const bool g = wait_bounded<true>(ptx::smem_u32(red_go), 0, abort_flag);
                    if (ptx::bar_red_or(kEpiBarrier, kEpiThreads, !g)) { ok = false; break; }
                    const uint32_t rbase = ptx::map_to_rank(ptx::smem_u32(red_buf), 0) +
                                           (rank * slot_words + (uint32_t)(i * BN)) * 4;
                    publish_row(nullptr, rbase, true);
                    ptx::mbar_arrive_remote(ptx::map_to_rank(ptx::smem_u32(red_full), 0));
                } else {
                    if (first_epi)
                        for (int r = 1; r < a.csplit; ++r) ptx::mbar_arrive_remote(ptx::map_to_rank(ptx::smem_u32(red_go), (uint32_t)r));
#pragma unroll
                    for (int c0 = 0; c0 < BN; c0 += 16) {
                        if (c0 >= ncv) break;
                        uint32_t v[16];
                        fetch16(c0, v);
                        if (has_row)
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj) red_buf[i * BN + c0 + jj] = v[jj];
                    }
                    ptx::bar_sync(kEpiBarrier, kEpiThreads);
                    const bool w = wait_bounded<true>(ptx::smem_u32(red_full), 0, abort_flag);
                    if (ptx::bar_red_or(kEpiBarrier, kEpiThreads, !w)) { ok = false; break; }
                    for (int col = te; col < ncv; col += kEpiThreads)
                        for (int r = 0; r < nrows; ++r) {
                            uint32_t v = red_buf[r * BN + col];
                            for (int k = 1; k < a.csplit; ++k)
                                v = add_words<KIND>(v, red_buf[k * slot_words + r * BN + col]);
                            finish(r, col, v);
                        }
                }
            } else if (kCompact && !full_tile) {
                // ---- partial, 64-row token tile: [row][column] words, one row per thread
                uint32_t* my = a.partials + ((size_t)blockIdx.x * 2 + slot) * (size_t)(BN * BM);
                publish_row(my + (size_t)(has_row ? i : 0) * BN, 0u, false);
            } else if (a.csplit > 1) {
                // ---- cluster split: ranks 1.. write their partial accumulators into rank
                // 0's shared memory (distributed shared memory) and arrive on its barrier;
                // rank 0 adds them in rank order, scales and stores.  The partials land in
                // rank 0's stage memory, so rank 0 first tells the others (remote arrive
                // on their `red_go`) that its MMAs -- the last readers of that memory --
                // have completed, which its accumulator being ready implies.
                const uint32_t rank = ptx::cluster_ctarank();
                if (rank != 0) {
                    const bool g = wait_bounded<true>(ptx::smem_u32(red_go), 0, abort_flag);
                    if (ptx::bar_red_or(kEpiBarrier, kEpiThreads, !g)) { ok = false; break; }
                    const uint32_t rbase = ptx::map_to_rank(ptx::smem_u32(red_buf), 0) +
                                           (rank - 1) * (uint32_t)(BN * BM * 4);
#pragma unroll
                    for (int c0 = 0; c0 < BN; c0 += 16) {
                        if (c0 >= ncv) break;
                        uint32_t v[16];
                        fetch16(c0, v);
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            if (c0 + jj < ncv && has_row) ptx::st_cluster_u32(rbase + (uint32_t)(((c0 + jj) * BM + i) * 4), v[jj]);
                    }
                    ptx::mbar_arrive_remote(ptx::map_to_rank(ptx::smem_u32(red_full), 0));
                } else {
                    if (first_epi)
                        for (int r = 1; r < a.csplit; ++r) ptx::mbar_arrive_remote(ptx::map_to_rank(ptx::smem_u32(red_go), (uint32_t)r));
                    const bool w = wait_bounded<true>(ptx::smem_u32(red_full), 0, abort_flag);
                    if (ptx::bar_red_or(kEpiBarrier, kEpiThreads, !w)) { ok = false; break; }
#pragma unroll
                    for (int c0 = 0; c0 < BN; c0 += 16) {
                        if (c0 >= ncv) break;
                        uint32_t v[16];
                        fetch16(c0, v);
                        for (int r = 1; r < a.csplit; ++r) {
                            const uint32_t* src = red_buf + (size_t)(r - 1) * (BN * BM);
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj)
                                v[jj] = add_words<BLOCK ? KIND_F8 : KIND>(v[jj], src[(c0 + jj) * BM + i]);
                        }
                        store_chunk16<KIND, BLOCK>(a, tokscale, r_row, c_base + c0, v, s_row, m_lo, m_hi);
                    }
                }
            } else if (full_tile) {
                // ---- whole K range in this CTA: scale and store
#pragma unroll
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    if (c0 >= ncv) break;
                    uint32_t v[16];
                    fetch16(c0, v);
                    store_chunk16<KIND, BLOCK>(a, tokscale, r_row, c_base + c0, v, s_row, m_lo, m_hi);
                }
            } else {
                // ---- partial: publish to this CTA's slot ([column][row] words, coalesced)
                uint32_t* my = a.partials + ((size_t)blockIdx.x * 2 + slot) * (size_t)(BN * BM);
#pragma unroll
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    if (c0 >= ncv) break;
                    uint32_t v[16];
                    fetch16(c0, v);
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj)
                        if (c0 + jj < ncv && has_row) __stcg(my + (size_t)(c0 + jj) * BM + i, v[jj]);
                }
            }
            if (!BLOCK) {
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(tempty + buf));
                if (++buf == kAccBufs) { buf = 0; bphase ^= 1u; }
            }
            if (!full_tile && a.csplit <= 1 && kCompact && a.pfix) {
                // ---- parallel fixup: count this contribution, finish the tile later
                __threadfence();
                ptx::bar_sync(kEpiBarrier, kEpiThreads);
                if (first_epi) atomicAdd(a.counters + t, 1);
                if (nfix < 2) fix_t[nfix] = t;
                ++nfix;
            } else if (!full_tile && a.csplit <= 1) {
                // ---- ticket: the last contributor of tile t finishes it
                __threadfence();
                ptx::bar_sync(kEpiBarrier, kEpiThreads);
                if (first_epi) *ticket = atomicAdd(a.counters + t, 1);
                ptx::bar_sync(kEpiBarrier, kEpiThreads);
                const int g_lo = cta_of_unit(a, (long long)t * nsb, U, Gp);
                const int g_hi = cta_of_unit(a, (long long)t * nsb + nsb - 1, U, Gp);
                if (*ticket == g_hi - g_lo && kCompact) {
                    // column-parallel: per column and row, contributors added in CTA order,
                    // four contributors' loads in flight together
                    __threadfence();
                    const int nc = g_hi - g_lo + 1;
                    for (int col = te; col < ncv; col += kEpiThreads)
                        for (int r0 = 0; r0 < nrows; r0 += 8) {
                            // 8 rows x 4 contributors of loads in flight per round trip
                            uint32_t v[8];
#pragma unroll
                            for (int rr = 0; rr < 8; ++rr) v[rr] = 0u;
                            for (int cb = 0; cb < nc; cb += 4) {
                                uint32_t x[4][8];
#pragma unroll
                                for (int k = 0; k < 4; ++k) {
                                    const int c = g_lo + cb + k;
                                    const uint32_t* p = nullptr;
                                    if (cb + k < nc) {
                                        const int sl = (unit_begin(a, c, U, Gp) / nsb == t) ? 0 : 1;
                                        p = a.partials + ((size_t)c * 2 + sl) * (size_t)(BN * BM) + col;
                                    }
#pragma unroll
                                    for (int rr = 0; rr < 8; ++rr)
                                        x[k][rr] = (p != nullptr && r0 + rr < nrows) ? __ldcg(p + (size_t)(r0 + rr) * BN) : 0u;
                                }
#pragma unroll
                                for (int k = 0; k < 4; ++k)
                                    if (cb + k < nc)
#pragma unroll
                                        for (int rr = 0; rr < 8; ++rr)
                                            v[rr] = (cb + k == 0) ? x[k][rr] : add_words<KIND>(v[rr], x[k][rr]);
                            }
#pragma unroll
                            for (int rr = 0; rr < 8; ++rr)
                                if (r0 + rr < nrows) finish(r0 + rr, col, v[rr]);
                        }
                    if (first_epi) a.counters[t] = 0;   // leave the counter ready for the next call
                } else if (*ticket == g_hi - g_lo) {
                    __threadfence();
                    const int nc = g_hi - g_lo + 1;
#pragma unroll 1
                    for (int c0 = 0; c0 < ncv; c0 += 16) {
                        uint32_t v[16];
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) v[jj] = 0u;
                        // contributors four at a time (their loads in flight together),
                        // added in CTA order, which fixes the summation order
#pragma unroll 1
                        for (int cb = 0; cb < nc; cb += 4) {
                            uint32_t x[4][16];
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const int c = g_lo + cb + k;
                                if (cb + k < nc) {
                                    const int sl = (unit_begin(a, c, U, Gp) / nsb == t) ? 0 : 1;
                                    const uint32_t* p = a.partials + ((size_t)c * 2 + sl) * (size_t)(BN * BM);
#pragma unroll
                                    for (int jj = 0; jj < 16; ++jj)
                                        x[k][jj] = (c0 + jj < ncv && has_row) ? __ldcg(p + (size_t)(c0 + jj) * BM + i) : 0u;
                                }
                            }
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                if (cb + k < nc) {
#pragma unroll
                                    for (int jj = 0; jj < 16; ++jj)
                                        v[jj] = (cb + k == 0) ? x[k][jj] : add_words<BLOCK ? KIND_F8 : KIND>(v[jj], x[k][jj]);
                                }
                            }
                        }
                        store_chunk16<KIND, BLOCK>(a, tokscale, r_row, c_base + c0, v, s_row, m_lo, m_hi);
                    }
                    if (first_epi) a.counters[t] = 0;   // leave the counter ready for the next call
                }
            }
            u += sb_hi - sb_lo;
        }
        if (BM == 64 && a.pfix && ok) {
            // ---- parallel fixup.  Every contributor of a split tile has published its
            // [row][column] partial before it waits here, so the waits end once the last
            // one has published.  Contributor j of nc adds, for its slice of 4-column
            // groups, the nc partials in CTA order; a second round of increments tells
            // the last one out to reset the counter for the next call.
            const int te = threadIdx.x - 64;
            for (int f = 0; f < nfix && f < 2; ++f) {
                const int t = fix_t[f];
                const int rt = t / a.c_tiles, ct = t % a.c_tiles;
                const int g_lo = cta_of_unit(a, (long long)t * nsb, U, Gp);
                const int g_hi = cta_of_unit(a, (long long)t * nsb + nsb - 1, U, Gp);
                const int nc = g_hi - g_lo + 1;
                const int j = (int)blockIdx.x - g_lo;
                bool w = true;
                if (first_epi) w = wait_count(a.counters + t, nc, abort_flag);
                if (ptx::bar_red_or(kEpiBarrier, kEpiThreads, !w)) { ok = false; break; }
                const int ncv = (a.rows_C - ct * BN < BN) ? a.rows_C - ct * BN : BN;
                const int nrows = (a.rows_R - rt * BM < BM) ? a.rows_R - rt * BM : BM;
                const int ng = (ncv + 3) / 4;
                const int gl = j * ng / nc, gw = (j + 1) * ng / nc - gl;
                for (int it = te; it < nrows * gw; it += kEpiThreads) {
                    const int r = it / gw, cg = gl + it % gw;
                    uint32_t v[4] = {0u, 0u, 0u, 0u};
                    for (int cb = 0; cb < nc; cb += 8) {
                        uint4 x[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const int c = g_lo + cb + k;
                            if (cb + k < nc) {
                                const int sl = (unit_begin(a, c, U, Gp) / nsb == t) ? 0 : 1;
                                const uint32_t* p = a.partials + ((size_t)c * 2 + sl) * (size_t)(BN * BM) +
                                                    (size_t)r * BN + 4 * cg;
                                x[k] = __ldcg(reinterpret_cast<const uint4*>(p));
                            }
                        }
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            if (cb + k < nc) {
                                const bool first = (cb + k == 0);
                                v[0] = first ? x[k].x : add_words<KIND>(v[0], x[k].x);
                                v[1] = first ? x[k].y : add_words<KIND>(v[1], x[k].y);
                                v[2] = first ? x[k].z : add_words<KIND>(v[2], x[k].z);
                                v[3] = first ? x[k].w : add_words<KIND>(v[3], x[k].w);
                            }
                        }
                    }
                    const int m = rt * BM + r;
                    const float sr = (a.out_i32 == nullptr) ? __ldg(a.sA + m) : 1.0f;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        if (4 * cg + q4 < ncv) store_out<KIND, BLOCK>(a, tokscale, m, ct * BN + 4 * cg + q4, v[q4], sr);
                }
                ptx::bar_sync(kEpiBarrier, kEpiThreads);
                if (first_epi && atomicAdd(a.counters + t, 1) == 2 * nc - 1) a.counters[t] = 0;
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}


struct GemmMaps {
    CUtensorMap R, C;
    int* occupancy = nullptr;   // when set: report resident CTAs per SM instead of launching
};

template <int BM, int BN, int KIND, bool BLOCK, int KPS, bool FQ = false, bool GRP = false>
cudaError_t launch_one(const GemmPlan& p, const GemmMaps& maps, const GemmArgs& args, cudaStream_t s)
{
    auto kern = gemm_kernel<BM, BN, KIND, BLOCK, KPS, FQ, GRP>;
    // the large dynamic shared-memory limit is a per-device function attribute
    static bool configured[64] = {};
    static std::mutex mu;
    {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
        std::lock_guard<std::mutex> lk(mu);
        if (!configured[dev]) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
            if (e != cudaSuccess) return e;
            configured[dev] = true;
        }
    }
    if (maps.occupancy != nullptr)
        return cudaOccupancyMaxActiveBlocksPerMultiprocessor(maps.occupancy, kern, kThreads, p.smem_bytes);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.G);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = p.smem_bytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (p.pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (p.cluster) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)p.split;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kern, maps.R, maps.C, args);
}


// Host accessor of this translation unit's device status word (defined once per unit
// that includes this header).
inline int status_word(int clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return W8_ERR_CUDA;
    if (clear && v != 0) {
        const int z = 0;
        if (cudaMemcpyToSymbol(g_device_status, &z, sizeof(int)) != cudaSuccess) return W8_ERR_CUDA;
    }
    return v;
}

// per-family launchers (one translation unit each)
cudaError_t launch_f8(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s);
cudaError_t launch_i8(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s);
cudaError_t launch_block(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s);
cudaError_t launch_bm64(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s);
cudaError_t launch_fq(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s);
cudaError_t launch_grouped(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s);
cudaError_t launch_pair(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s);
cudaError_t launch_decode(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s);
int status_f8(int clear);
int status_i8(int clear);
int status_block(int clear);
int status_bm64(int clear);
int status_fq(int clear);
int status_grouped(int clear);
int status_pair(int clear);
int status_decode(int clear);

}  // namespace gemm
}  // namespace w8
