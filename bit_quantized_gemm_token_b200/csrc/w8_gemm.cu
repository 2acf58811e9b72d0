// w8_gemm.cu -- the scaled 8-bit GEMM: one sm_100a kernel family (tcgen05 MMA, TMEM
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
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "w8_internal.h"
#include "w8_ptx.cuh"

namespace w8 {

__device__ int g_device_status;   // first device-side error (0 = none)

namespace {

constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kEpiBarrier = 1;          // named barrier id of the epilogue warps
constexpr int kRBytes = 128 * 128;      // one R tile: 128 rows x 128 K-bytes
constexpr int kNumAcc = 2;              // TMEM accumulator buffers
constexpr unsigned long long kWaitNs = 1000000000ull;   // 1 s bound on any single wait

enum { KIND_F8 = 0, KIND_I8 = 1 };

struct GemmArgs {
    int M, N, K;
    int swap;
    int rows_R, rows_C;
    int r_tiles, c_tiles, tiles, kbs;
    long long units;
    int G;
    int align_tiles;
    int stages;
    int pdl;
    int ld_sblk;   // K/128: row length of the block-scale matrices
    int vec_ok;    // Standard epilogue may use 16-byte stores (N % 8 == 0, out 16-byte aligned)
    const float* sA;
    const float* sW;
    __nv_bfloat16* out;
    int32_t* out_i32;
    uint32_t* partials;   // [G][2][BN][128] raw fp32 / int32 words
    int* counters;        // [tiles]
};

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
// K-major, M = 128, N = BN.
template <int KIND, int BN>
__device__ __forceinline__ constexpr uint32_t instr_desc()
{
    return (KIND == KIND_I8 ? (2u << 4) : (1u << 4))      // bits 4-5: D format
           | (KIND == KIND_I8 ? (1u << 7) : 0u)           // bits 7-9: A format (s8 / e4m3)
           | (KIND == KIND_I8 ? (1u << 10) : 0u)          // bits 10-12: B format
           | ((uint32_t)(BN >> 3) << 17)                  // bits 17-22: N / 8
           | ((uint32_t)(128 >> 4) << 24);                // bits 24-28: M / 16
}

// ---------------------------------------------------------------- unit partition
__device__ __forceinline__ long long unit_begin(const GemmArgs& a, long long g)
{
    if (a.align_tiles) return (g * a.tiles / a.G) * a.kbs;
    return g * a.units / a.G;
}

__device__ __forceinline__ int cta_of_unit(const GemmArgs& a, long long u)
{
    return (int)(((u + 1) * (long long)a.G - 1) / a.units);
}

// ---------------------------------------------------------------- bounded waits
__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_device_status, 0, code); }

// Poll an mbarrier phase until it completes, the deadline passes, or another role of
// this CTA has given up (abort flag).  Returns false on give-up.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag)
{
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 0) {
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
template <int KIND, bool BLOCK>
__device__ __forceinline__ void store_out(const GemmArgs& a, int r_row, int c_row, uint32_t w, float s_row)
{
    const int m = a.swap ? c_row : r_row;
    const int n = a.swap ? r_row : c_row;
    if (m >= a.M || n >= a.N) return;
    const size_t o = (size_t)m * a.N + n;
    if (KIND == KIND_I8 && a.out_i32 != nullptr) {
        a.out_i32[o] = (int32_t)w;
        return;
    }
    float v = word_to_float<KIND>(w);
    if (!BLOCK) {
        // s_row is the scale of the R-side index; the C-side scale is looked up here
        const float s_col = a.swap ? __ldg(a.sA + m) : __ldg(a.sW + n);
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
__device__ __forceinline__ void store_chunk16(const GemmArgs& a, int r_row, int c_base, const uint32_t (&v)[16],
                                              float s_row)
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
    for (int jj = 0; jj < 16; ++jj) store_out<KIND, BLOCK>(a, r_row, c_base + jj, v[jj], s_row);
}

// ---------------------------------------------------------------- the kernel
template <int BN, int KIND, bool BLOCK>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmC, const GemmArgs a)
{
    constexpr int kCBytes = BN * 128;
    constexpr int kStageBytes = kRBytes + kCBytes;
    constexpr uint32_t kTmemCols = (kNumAcc * BN <= 32) ? 32 : (kNumAcc * BN <= 64) ? 64 : (kNumAcc * BN <= 128) ? 128 : (kNumAcc * BN <= 256) ? 256 : 512;
    constexpr uint32_t kIdesc = instr_desc<KIND, BN>();

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = a.stages;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * kStageBytes);
    uint64_t* empty = full + S;
    uint64_t* tfull = empty + S;
    uint64_t* tempty = tfull + kNumAcc;
    uint64_t* drain = tempty + kNumAcc;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* ticket = reinterpret_cast<volatile int*>(tmem_slot + 2);

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
        *abort_flag = 0;
        ptx::fence_barrier_init();
    }
    if (threadIdx.x == 32) {
        ptx::prefetch_tmap(&tmR);
        ptx::prefetch_tmap(&tmC);
    }
    if (warp == 1) ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const long long u0 = unit_begin(a, blockIdx.x);
    const long long u1 = unit_begin(a, blockIdx.x + 1);
    const int kbs = a.kbs;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_w = ptx::policy_evict_first();   // weights: streamed once
            const uint64_t pol_a = ptx::policy_evict_last();    // activations: re-read by every CTA
            const uint64_t pol_R = a.swap ? pol_w : pol_a;
            const uint64_t pol_C = a.swap ? pol_a : pol_w;
            const long long n = u1 - u0;
            // With programmatic dependent launch the weight tiles of the first `pre`
            // stages are requested before waiting for the previous kernel (weights are
            // never its output); the activation tiles follow after the wait.
            const int pre = a.pdl ? (int)(n < S ? n : S) : 0;
            for (int i = 0; i < pre; ++i) {
                const long long u = u0 + i;
                const int t = (int)(u / kbs), kb = (int)(u % kbs);
                const int rt = t / a.c_tiles, ct = t % a.c_tiles;
                uint8_t* st = smem + (size_t)i * kStageBytes;
                const uint32_t fb = ptx::smem_u32(full + i);
                ptx::mbar_arrive_expect_tx(fb, kStageBytes);
                if (a.swap) ptx::tma_load_2d(ptx::smem_u32(st), &tmR, fb, kb * 128, rt * 128, pol_R);
                else        ptx::tma_load_2d(ptx::smem_u32(st + kRBytes), &tmC, fb, kb * 128, ct * BN, pol_C);
            }
            ptx::grid_dep_wait();
            ptx::grid_dep_launch();
            for (int i = 0; i < pre; ++i) {
                const long long u = u0 + i;
                const int t = (int)(u / kbs), kb = (int)(u % kbs);
                const int rt = t / a.c_tiles, ct = t % a.c_tiles;
                uint8_t* st = smem + (size_t)i * kStageBytes;
                const uint32_t fb = ptx::smem_u32(full + i);
                if (a.swap) ptx::tma_load_2d(ptx::smem_u32(st + kRBytes), &tmC, fb, kb * 128, ct * BN, pol_C);
                else        ptx::tma_load_2d(ptx::smem_u32(st), &tmR, fb, kb * 128, rt * 128, pol_R);
            }
            long long issued = pre;
            int stage = pre % S;
            uint32_t phase = (pre == S) ? 1u : 0u;
            for (long long i = pre; i < n; ++i) {
                const long long u = u0 + i;
                const int t = (int)(u / kbs), kb = (int)(u % kbs);
                const int rt = t / a.c_tiles, ct = t % a.c_tiles;
                if (!wait_bounded(ptx::smem_u32(empty + stage), phase ^ 1u, abort_flag)) break;
                uint8_t* st = smem + (size_t)stage * kStageBytes;
                const uint32_t fb = ptx::smem_u32(full + stage);
                ptx::mbar_arrive_expect_tx(fb, kStageBytes);
                ptx::tma_load_2d(ptx::smem_u32(st), &tmR, fb, kb * 128, rt * 128, pol_R);
                ptx::tma_load_2d(ptx::smem_u32(st + kRBytes), &tmC, fb, kb * 128, ct * BN, pol_C);
                ++issued;
                if (++stage == S) { stage = 0; phase ^= 1u; }
            }
            if (*abort_flag) {
                // let the copies still in flight land before the CTA unwinds: the last
                // min(S, issued) loads (earlier ones were consumed), each bounded
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
        int stage = 0, buf = 0;
        uint32_t phase = 0, bphase = 0;
        bool ok = true;
        for (long long u = u0; u < u1 && ok; ++u) {
            const int kb = (int)(u % kbs);
            const bool first = BLOCK || u == u0 || kb == 0;
            const bool last = BLOCK || u == u1 - 1 || kb == kbs - 1;
            if (lane == 0) {
                if (first) {
                    ok = wait_bounded(ptx::smem_u32(tempty + buf), bphase ^ 1u, abort_flag);
                    ptx::tc_fence_after();
                }
                if (ok) ok = wait_bounded(ptx::smem_u32(full + stage), phase, abort_flag);
                if (ok) {
                    ptx::tc_fence_after();
                    const uint8_t* st = smem + (size_t)stage * kStageBytes;
                    const uint64_t dR = smem_desc(ptx::smem_u32(st));
                    const uint64_t dC = smem_desc(ptx::smem_u32(st + kRBytes));
                    const uint32_t d_tmem = tmem + (uint32_t)(buf * BN);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        // advance 32 K-bytes inside the 128-byte swizzle row: +2 in 16-byte units
                        const uint32_t acc = (first && k == 0) ? 0u : 1u;
                        if (KIND == KIND_I8) ptx::mma_i8(d_tmem, dR + 2 * k, dC + 2 * k, kIdesc, acc);
                        else                 ptx::mma_f8f6f4(d_tmem, dR + 2 * k, dC + 2 * k, kIdesc, acc);
                    }
                    ptx::mma_commit(ptx::smem_u32(empty + stage));
                    if (last) ptx::mma_commit(ptx::smem_u32(tfull + buf));
                }
            }
            ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
            if (++stage == S) { stage = 0; phase ^= 1u; }
            if (last) {
                if (++buf == kNumAcc) { buf = 0; bphase ^= 1u; }
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
        ptx::grid_dep_wait();
        const int q = warp & 3;                 // TMEM lane quadrant of this warp
        const int i = q * 32 + lane;            // row of the R tile held by this thread
        const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
        const bool first_epi = (threadIdx.x == 64);
        constexpr int kAccRegs = BLOCK ? BN : 1;
        int buf = 0;
        uint32_t bphase = 0;
        bool ok = true;
        for (long long u = u0; u < u1 && ok;) {
            const int t = (int)(u / kbs);
            const int kb_lo = (int)(u % kbs);
            const long long rem = u1 - u;
            const int kb_hi = (int)((kbs - kb_lo < rem) ? kbs : kb_lo + rem);
            const int rt = t / a.c_tiles, ct = t % a.c_tiles;
            const int r_row = rt * 128 + i;
            const bool full_tile = (kb_lo == 0 && kb_hi == kbs);
            const int slot = (u == u0) ? 0 : 1;
            // scale of this thread's R-side index (FP8 / INT8; BLOCK scales per K block)
            float s_row = 1.0f;
            if (!BLOCK && a.out_i32 == nullptr && r_row < a.rows_R) s_row = __ldg((a.swap ? a.sW : a.sA) + r_row);

            float acc[kAccRegs];
#pragma unroll
            for (int j = 0; j < kAccRegs; ++j) acc[j] = 0.0f;
            if (BLOCK) {
                // ---- per-K-block promotion: acc += (sA * sW) * (block dot product), fp32
                for (int kb = kb_lo; kb < kb_hi; ++kb) {
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
                            sa_l[h] = (jc < BN && col < a.rows_C) ? __ldg(a.sA + (size_t)col * a.ld_sblk + kb) : 0.0f;
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
                    if (++buf == kNumAcc) { buf = 0; bphase ^= 1u; }
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

            if (full_tile) {
                // ---- whole K range in this CTA: scale and store
#pragma unroll
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    uint32_t v[16];
                    fetch16(c0, v);
                    store_chunk16<KIND, BLOCK>(a, r_row, ct * BN + c0, v, s_row);
                }
            } else {
                // ---- partial: publish to this CTA's slot ([column][row] words, coalesced)
                uint32_t* my = a.partials + ((size_t)blockIdx.x * 2 + slot) * (size_t)(BN * 128);
#pragma unroll
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    uint32_t v[16];
                    fetch16(c0, v);
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) __stcg(my + (size_t)(c0 + jj) * 128 + i, v[jj]);
                }
            }
            if (!BLOCK) {
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(tempty + buf));
                if (++buf == kNumAcc) { buf = 0; bphase ^= 1u; }
            }
            if (!full_tile) {
                // ---- ticket: the last contributor of tile t finishes it
                __threadfence();
                ptx::bar_sync(kEpiBarrier, kEpiThreads);
                if (first_epi) *ticket = atomicAdd(a.counters + t, 1);
                ptx::bar_sync(kEpiBarrier, kEpiThreads);
                const int g_lo = cta_of_unit(a, (long long)t * kbs);
                const int g_hi = cta_of_unit(a, (long long)t * kbs + kbs - 1);
                if (*ticket == g_hi - g_lo) {
                    __threadfence();
#pragma unroll 1
                    for (int c0 = 0; c0 < BN; c0 += 16) {
                        uint32_t v[16];
#pragma unroll 1
                        for (int c = g_lo; c <= g_hi; ++c) {   // fixed order: CTA index
                            const int sl = (unit_begin(a, c) / kbs == t) ? 0 : 1;
                            const uint32_t* p = a.partials + ((size_t)c * 2 + sl) * (size_t)(BN * 128);
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj) {
                                const uint32_t x = __ldcg(p + (size_t)(c0 + jj) * 128 + i);
                                v[jj] = (c == g_lo) ? x : add_words<BLOCK ? KIND_F8 : KIND>(v[jj], x);
                            }
                        }
                        store_chunk16<KIND, BLOCK>(a, r_row, ct * BN + c0, v, s_row);
                    }
                    if (first_epi) a.counters[t] = 0;   // leave the counter ready for the next call
                }
            }
            u += kb_hi - kb_lo;
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

// ================================================================ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Row-major byte matrix [rows, cols] viewed as a 2-D tensor, boxes of 128 bytes x box_rows
// rows, 128-byte swizzle; out-of-range boxes read zeros.
bool make_tmap(CUtensorMap* m, const void* base, int rows, int cols, int box_rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

constexpr int tile_bn(int id) { return 16 << id; }

size_t stage_bytes(int bn) { return (size_t)kRBytes + (size_t)bn * 128; }

size_t smem_for(int bn, int stages)
{
    return 1024 + (size_t)stages * stage_bytes(bn) + (size_t)(2 * stages + 2 * kNumAcc + 1) * 8 + 16;
}

int default_stages(int bn)
{
    switch (bn) {
    case 16: return 5;
    case 32: return 5;
    case 64: return 4;
    case 128: return 6;
    default: return 4;
    }
}

template <int BN, int KIND, bool BLOCK>
cudaError_t launch_one(const GemmPlan& p, const CUtensorMap& tR, const CUtensorMap& tC, const GemmArgs& args,
                       cudaStream_t s)
{
    auto kern = gemm_kernel<BN, KIND, BLOCK>;
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
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.G);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = p.smem_bytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, tR, tC, args);
}

}  // namespace

// ---------------------------------------------------------------- planning
int gemm_plan(int fmt, int M, int N, int K, int variant, int sm_count, GemmPlan* p)
{
    if (M <= 0 || N <= 0 || K <= 0) return W8_ERR_INVALID_ARG;
    if (fmt < W8_FMT_FP8_DYN || fmt > W8_FMT_BLOCK_FP8_UE8M0) return W8_ERR_INVALID_ARG;
    const bool block = fmt >= W8_FMT_BLOCK_FP8;
    if (K % 16 != 0) return W8_ERR_ALIGNMENT;
    if (block && K % 128 != 0) return W8_ERR_ALIGNMENT;
    if (!(variant & W8_V_EXPLICIT)) return W8_ERR_INVALID_ARG;   // AUTO is resolved by the caller

    GemmPlan q = {};
    q.fmt = fmt;
    q.M = M; q.N = N; q.K = K;
    q.swap = (variant & W8_V_SWAP_AB) ? 1 : 0;
    q.stream = (variant & W8_V_STREAM) ? 1 : 0;
    const int lg = (variant >> W8_V_SPLIT_SHIFT) & 0xF;
    const int tid = (variant >> W8_V_TILE_SHIFT) & 0xF;
    int stages = (variant >> W8_V_STAGES_SHIFT) & 0xF;
    q.pdl = (variant & W8_V_PDL) ? 1 : 0;
    if (lg > 8) return W8_ERR_UNSUPPORTED;
    if (tid >= kNumTiles) return W8_ERR_UNSUPPORTED;
    q.bn = tile_bn(tid);
    if (block && q.bn > 64) return W8_ERR_UNSUPPORTED;   // block promotion keeps the tile in registers
    q.split = 1 << lg;
    if (stages == 0) stages = default_stages(q.bn);
    if (stages < 2) return W8_ERR_UNSUPPORTED;
    q.stages = stages;
    q.smem_bytes = smem_for(q.bn, stages);
    if (q.smem_bytes > 232448) return W8_ERR_UNSUPPORTED;

    q.rows_R = q.swap ? N : M;
    q.rows_C = q.swap ? M : N;
    q.r_tiles = (q.rows_R + 127) / 128;
    q.c_tiles = (q.rows_C + q.bn - 1) / q.bn;
    q.tiles = q.r_tiles * q.c_tiles;
    q.kbs = (K + 127) / 128;
    q.units = (long long)q.tiles * q.kbs;
    if (q.stream) {
        long long g = sm_count > 0 ? sm_count : 148;
        if (g > q.units) g = q.units;
        q.G = (int)g;
        q.align_tiles = 0;
    } else if (q.split > 1) {
        if (q.split > q.kbs) return W8_ERR_UNSUPPORTED;
        const long long g = (long long)q.tiles * q.split;
        if (g > 0x7FFFFFFF) return W8_ERR_UNSUPPORTED;
        q.G = (int)g;
        q.align_tiles = 0;
    } else {
        int g = sm_count > 0 ? sm_count : 148;
        if (g > q.tiles) g = q.tiles;
        q.G = g;
        q.align_tiles = 1;
    }
    // partial slots exist whenever some tile's K range can be split across CTAs
    const bool partials = !q.align_tiles && !(q.G == q.tiles);   // G == tiles with stream: one CTA per tile
    if (partials) {
        q.ws_counters = (((size_t)q.tiles * 4) + 255) & ~(size_t)255;
        q.ws_bytes = q.ws_counters + (size_t)q.G * 2 * (size_t)q.bn * 128 * 4;
    } else {
        q.ws_counters = 0;
        q.ws_bytes = 0;
    }
    *p = q;
    return W8_OK;
}

// ---------------------------------------------------------------- launch
int gemm_launch(const GemmPlan& p, const void* A_q, const float* A_scale, const void* W_q, const float* W_scale,
                void* out, int32_t* out_i32, void* workspace, size_t ws_bytes, cudaStream_t s)
{
    if (p.ws_bytes > 0 && (workspace == nullptr || ws_bytes < p.ws_bytes)) return W8_ERR_WORKSPACE;
    if (p.ws_bytes > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255)) return W8_ERR_ALIGNMENT;
    CUtensorMap tR, tC;
    const void* R = p.swap ? W_q : A_q;
    const void* C = p.swap ? A_q : W_q;
    if (!make_tmap(&tR, R, p.rows_R, p.K, 128)) return W8_ERR_CUDA;
    if (!make_tmap(&tC, C, p.rows_C, p.K, p.bn)) return W8_ERR_CUDA;

    GemmArgs args = {};
    args.M = p.M; args.N = p.N; args.K = p.K;
    args.swap = p.swap;
    args.rows_R = p.rows_R; args.rows_C = p.rows_C;
    args.r_tiles = p.r_tiles; args.c_tiles = p.c_tiles; args.tiles = p.tiles; args.kbs = p.kbs;
    args.units = p.units;
    args.G = p.G;
    // no workspace means every CTA range is made of whole tiles
    args.align_tiles = (p.align_tiles || p.ws_bytes == 0) ? 1 : 0;
    args.stages = p.stages;
    args.pdl = p.pdl;
    args.ld_sblk = p.kbs;
    args.sA = A_scale;
    args.sW = W_scale;
    args.out = static_cast<__nv_bfloat16*>(out);
    args.out_i32 = out_i32;
    args.counters = p.ws_bytes ? static_cast<int*>(workspace) : nullptr;
    args.partials = p.ws_bytes ? reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + p.ws_counters) : nullptr;
    args.vec_ok = (p.N % 8 == 0) && ((reinterpret_cast<uintptr_t>(out) & 15) == 0);

    const bool block = p.fmt >= W8_FMT_BLOCK_FP8;
    const bool i8 = p.fmt == W8_FMT_INT8;
    cudaError_t e = cudaErrorInvalidValue;
    if (block) {
        switch (p.bn) {
        case 16: e = launch_one<16, KIND_F8, true>(p, tR, tC, args, s); break;
        case 32: e = launch_one<32, KIND_F8, true>(p, tR, tC, args, s); break;
        case 64: e = launch_one<64, KIND_F8, true>(p, tR, tC, args, s); break;
        default: return W8_ERR_UNSUPPORTED;
        }
    } else if (i8) {
        switch (p.bn) {
        case 16: e = launch_one<16, KIND_I8, false>(p, tR, tC, args, s); break;
        case 32: e = launch_one<32, KIND_I8, false>(p, tR, tC, args, s); break;
        case 64: e = launch_one<64, KIND_I8, false>(p, tR, tC, args, s); break;
        case 128: e = launch_one<128, KIND_I8, false>(p, tR, tC, args, s); break;
        case 256: e = launch_one<256, KIND_I8, false>(p, tR, tC, args, s); break;
        default: return W8_ERR_UNSUPPORTED;
        }
    } else {
        switch (p.bn) {
        case 16: e = launch_one<16, KIND_F8, false>(p, tR, tC, args, s); break;
        case 32: e = launch_one<32, KIND_F8, false>(p, tR, tC, args, s); break;
        case 64: e = launch_one<64, KIND_F8, false>(p, tR, tC, args, s); break;
        case 128: e = launch_one<128, KIND_F8, false>(p, tR, tC, args, s); break;
        case 256: e = launch_one<256, KIND_F8, false>(p, tR, tC, args, s); break;
        default: return W8_ERR_UNSUPPORTED;
        }
    }
    return e == cudaSuccess ? W8_OK : W8_ERR_CUDA;
}

int gemm_device_status(int clear)
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return W8_ERR_CUDA;
    if (clear) {
        const int z = 0;
        if (cudaMemcpyToSymbol(g_device_status, &z, sizeof(int)) != cudaSuccess) return W8_ERR_CUDA;
    }
    return v;
}

}  // namespace w8
