// w8_gemm_decode.cu -- the decode form of the scaled 8-bit GEMM (M <= 64 tokens),
// FP8-dynamic and W8A8-INT8.
//
// What it computes is the Standard form's sum ("Helion DSL added to vLLM to autotune
// linear inference backends", section "Unified GEMM Architecture"; "Helion nel backend
// vLLM: un solo GEMM ...", paragraphs 2-3, Split-K):
//   out[m, n] = bf16( (sum_k A[m,k] W[n,k]) * sA[m] * sW[n] ),
// with the K range cut into C contiguous chunks whose fp32 (int32 for INT8) partial sums
// are added in chunk order -- a Split-K with C = 1..8 chunks.
//
// How it is laid out on the B200:
//  * Operands.  The tokens occupy the tensor core's 64-row operand and the weights its
//    wide one: BN weight rows (64..256, a multiple of 16) per MMA.  A tcgen05.mma costs
//    about the same time whatever its N, so each one consumes BN x 32 weight bytes --
//    8 KB at BN = 256, twice what a 128-row weight operand gives -- and the tensor core
//    runs well ahead of HBM instead of just keeping up with it.
//  * Shared memory.  A stage holds the token box (M rounded up to 8 rows x 128 bytes)
//    followed by the weight box (BN rows).  The MMA reads 64 token rows; the ones past
//    the box lie in the stage's weight box and only feed accumulator rows that are never
//    stored (row m of the product depends on row m of the token operand alone).  With
//    three stages a CTA needs at most ~110 KB and fewer than 170 registers per thread,
//    so a CTA of the next GEMM on the stream fits beside one of this GEMM on the same
//    SM: under programmatic dependent launch it loads its first weight stages while
//    this one finishes.
//  * Grid.  ceil(N / BN) weight tiles x C K chunks; the C CTAs of a tile form one
//    thread-block cluster (rank r takes K blocks [r kbs / C, (r+1) kbs / C)).
//  * Reduction.  A reduce-scatter through distributed shared memory: rank r finishes
//    the columns [r SW, (r+1) SW) of the tile.  Once every rank's MMAs are done (each
//    tells the others), every rank writes each owner its partial sums of the owner's
//    columns with st.async into the owner's stage memory; each owner adds the C partials
//    of every element in rank order, scales and stores.  The tail never goes through
//    global memory.
//  * Weight stream.  The producer keeps `l2ahead` K blocks of weights in flight into L2
//    (bulk tensor prefetch) ahead of the shared-memory stages.
//
// Per CTA (192 threads): warp 0 = TMA producer, warp 1 = TMEM allocator + MMA issuer,
// warps 2..5 = epilogue.  The accumulator of a 64-row MMA keeps row r in TMEM lane
// (r % 16) + 32 (r / 16): epilogue warp w reads the tokens 16 (w % 4) .. + 15.  Every
// wait is bounded by the global timer (W8_ERR_DEVICE_TIMEOUT in the device status word).
#include "w8_gemm_kernel.cuh"

namespace w8 {
namespace gemm {
namespace {

__host__ __device__ constexpr uint32_t decode_idesc(int kind, int bn)
{
    return (kind == KIND_I8 ? (2u << 4) : (1u << 4))            // D format: s32 / f32
           | (kind == KIND_I8 ? ((1u << 7) | (1u << 10)) : 0u)  // A, B formats: s8 / e4m3
           | ((uint32_t)(bn >> 3) << 17)                        // N / 8
           | ((uint32_t)(64 >> 4) << 24);                       // M / 16
}

__device__ __forceinline__ uint32_t tmem_cols_for(int bn)
{
    return bn <= 32 ? 32u : bn <= 64 ? 64u : bn <= 128 ? 128u : 256u;
}

// Bounded spin on a local barrier phase that ignores the abort flag (unwinding).
__device__ __forceinline__ void settle_local(uint32_t bar, uint32_t parity)
{
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(bar, parity) && ptx::globaltimer_ns() - t0 < 10000000ull) {}
}

template <int KIND, bool FQ>
__global__ void __launch_bounds__(kThreads, 2)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                       const GemmArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem_base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = a.stages;
    const int BN = a.bn;
    const int m8 = a.m8;
    const int C = a.csplit;
    const int M = a.M;
    // FQ: the token codes of this rank's K blocks ([K block][m8 rows][128 bytes], 128-byte
    // swizzled as a TMA box would land), then stages that carry weight boxes only
    uint8_t* a_region = smem_base;
    uint8_t* smem = smem_base + (FQ ? a.a_region : 0);
    const size_t stage_bytes = (size_t)((FQ ? 0 : m8) + BN) * 128;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * stage_bytes);
    uint64_t* empty = full + S;
    uint64_t* tfull = empty + S;     // the accumulator is complete
    uint64_t* freeb = tfull + 1;     // C > 1: the other ranks' MMAs are done (their stages may receive)
    uint64_t* recvb = freeb + 1;     // C > 1: the other ranks' partials of this rank's columns landed
    uint64_t* drain = recvb + 1;
    uint64_t* a_ready = drain + 1;   // FQ: the token codes are in the region
    uint64_t* amaxb = a_ready + 1;   // FQ, C > 1: the other ranks' partial token maxima landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(FQ ? amaxb + 1 : drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* s_w = reinterpret_cast<float*>(tmem_slot + 4);   // [256] weight scales of this rank's columns
    float* s_a = s_w + 256;                                  // [64] token scales, then [8] words
    uint32_t* amax_slots = reinterpret_cast<uint32_t*>(s_a + 64 + 8);   // FQ: [8 ranks][64 tokens]
    auto a_slot = [&](int s) { return smem + (size_t)s * stage_bytes; };
    auto w_slot = [&](int s) { return smem + (size_t)s * stage_bytes + (FQ ? 0 : (size_t)m8 * 128); };
    const int SW = a.sw;
    const int RS = SW + 4;   // row stride in words: token rows fall on different banks

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tile = (int)blockIdx.x / C;
    const uint32_t rank = (C > 1) ? ptx::cluster_ctarank() : 0u;
    const int kbs = a.kbs;
    // rank r holds K blocks [r kbs / C, (r + 1) kbs / C): kbs / C or one more
    auto kb_first = [&](int r) { return r * kbs / C; };
    const int kb0 = kb_first((int)rank);
    const int nkb = kb_first((int)rank + 1) - kb0;
    const int n0 = tile * BN;
    // width of rank r's column share
    auto share = [&](int r) { return max(0, min(SW, BN - r * SW)); };
    const uint32_t tmem_cols = tmem_cols_for(BN);
    const uint64_t wlim = a.wait_ns ? a.wait_ns : kWaitNs;   // bound on every wait
    const int nload = a.starve ? 0 : nkb;                     // K blocks the producer loads
    // Receive area: [C source ranks][M tokens][RS words], the partial sums of the columns
    // this rank finishes.  It lies over the R consecutive stages whose last use comes
    // earliest, so that it is free -- and the other ranks may write into it -- a few K
    // blocks before this rank's last MMA.  Stage s last holds K block last_use(s).
    // The area spans R stages from stage recv_first[.]: the planner chose, for each of the
    // two K-block counts a rank can hold, the window of stages last used earliest (the
    // ranks may differ, so a sender looks up the receiver's).
    auto last_use = [&](int st, int n) { return st < n ? st + S * ((n - 1 - st) / S) : -1; };
    const size_t recv_bytes = (size_t)C * M * RS * 4;
    const int R = a.recv_R;
    auto recv_stage = [&](int r) {
        return (kb_first(r + 1) - kb_first(r)) == a.nkb_lo ? a.recv_first[0] : a.recv_first[1];
    };
    const int s0 = recv_stage((int)rank);
    uint32_t* recv = reinterpret_cast<uint32_t*>(smem + (size_t)s0 * stage_bytes);
    // Staging area: the accumulator rows [M][BN] copied out of tensor memory by the token
    // lanes, so that all 128 epilogue threads can then send them (each token lane alone
    // would issue BN / 4 remote stores); at the end of the stage memory, used only after
    // this rank's MMAs are done, never inside the receive area.  Without room for it the
    // token lanes send directly.
    const size_t stg_bytes = (size_t)M * BN * 4;
    const size_t stg_off = ((size_t)S * stage_bytes - stg_bytes) & ~(size_t)15;
    const bool use_stg = C > 1 && stg_bytes <= (size_t)S * stage_bytes &&
                         (size_t)s0 * stage_bytes + recv_bytes <= stg_off;
    uint32_t* stg = reinterpret_cast<uint32_t*>(smem + stg_off);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(ptx::smem_u32(full + s), 1);
            ptx::mbar_init(ptx::smem_u32(empty + s), 1);
        }
        ptx::mbar_init(ptx::smem_u32(tfull), 1);
        ptx::mbar_init(ptx::smem_u32(freeb), C > 1 ? (uint32_t)(C - 1) : 1u);
        ptx::mbar_init(ptx::smem_u32(recvb), 1);
        ptx::mbar_init(ptx::smem_u32(drain), 1);
        if (FQ) {
            ptx::mbar_init(ptx::smem_u32(a_ready), 1);
            ptx::mbar_init(ptx::smem_u32(amaxb), 1);
        }
        *abort_flag = 0;
        ptx::fence_barrier_init();
        // the bytes the other ranks will write into this rank's receive area
        if (C > 1) ptx::mbar_arrive_expect_tx(ptx::smem_u32(recvb), (uint32_t)((C - 1) * M * share((int)rank) * 4));
        // FQ: and their partial token maxima (m8 words each)
        if (FQ && C > 1) ptx::mbar_arrive_expect_tx(ptx::smem_u32(amaxb), (uint32_t)((C - 1) * m8 * 4));
    }
    if (threadIdx.x == 32) {
        ptx::prefetch_tmap(&tmA);
        ptx::prefetch_tmap(&tmW);
    }
    __syncthreads();
    // every rank's barriers are initialised before any rank signals another
    if (C > 1) ptx::cluster_sync();
    uint32_t tmem = 0;
    if (warp != 0) {
        if (warp == 1) {
            ptx::tmem_alloc(ptx::smem_u32(tmem_slot), tmem_cols);
            // dependents are released once this CTA holds its tensor memory (a CTA of the
            // next kernel on this SM can then never hold columns this one still needs)
            if (lane == 0) ptx::grid_dep_launch();
        }
        ptx::tc_fence_before();
        ptx::bar_sync(kTmemBarrier, kThreads - 32);
        ptx::tc_fence_after();
        tmem = *tmem_slot;
    }

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_w = ptx::policy_evict_first();   // weights: streamed once
            const uint64_t pol_a = ptx::policy_evict_last();    // tokens: read by every weight tile
            const uint32_t tx = (uint32_t)stage_bytes;
            const int D = a.l2ahead;
            // weights are never written by the work ahead of this kernel: under PDL the
            // first stages' weight boxes are requested before waiting for it
            const int pre = a.pdl ? min(nload, S) : 0;
            for (int i = 0; i < pre; ++i) {
                const uint32_t fb = ptx::smem_u32(full + i);
                ptx::mbar_arrive_expect_tx(fb, tx);
                ptx::tma_load_2d(ptx::smem_u32(w_slot(i)), &tmW, fb, (kb0 + i) * 128, n0, pol_w);
            }
            const int first = min(nload, S);   // K blocks whose loads go out without waiting for a stage
            for (int i = first; i < min(nload, first + D); ++i) ptx::tma_prefetch_l2_2d(&tmW, (kb0 + i) * 128, n0);
            ptx::grid_dep_wait();
            if (!FQ)
                for (int i = 0; i < pre; ++i)
                    ptx::tma_load_2d(ptx::smem_u32(a_slot(i)), &tmA, ptx::smem_u32(full + i), (kb0 + i) * 128, 0, pol_a);
            int stage = pre % S;
            uint32_t phase = (pre == S) ? 1u : 0u;
            int issued = pre;
            for (int i = pre; i < nload; ++i) {
                if (!wait_bounded(ptx::smem_u32(empty + stage), phase ^ 1u, abort_flag, wlim)) break;
                const uint32_t fb = ptx::smem_u32(full + stage);
                ptx::mbar_arrive_expect_tx(fb, tx);
                ptx::tma_load_2d(ptx::smem_u32(w_slot(stage)), &tmW, fb, (kb0 + i) * 128, n0, pol_w);
                if (!FQ) ptx::tma_load_2d(ptx::smem_u32(a_slot(stage)), &tmA, fb, (kb0 + i) * 128, 0, pol_a);
                if (i >= first && i + D < nload) ptx::tma_prefetch_l2_2d(&tmW, (kb0 + i + D) * 128, n0);
                ++issued;
                if (++stage == S) { stage = 0; phase ^= 1u; }
            }
            if (*abort_flag) {
                // the copies still in flight land before the CTA unwinds (bounded)
                for (int j = issued > S ? issued - S : 0; j < issued; ++j)
                    settle_local(ptx::smem_u32(full + (j % S)), (uint32_t)((j / S) & 1));
            } else if (C > 1) {
                // once the MMAs have read the receive area's stages for the last time, tell
                // every other rank that it may write its partial sums there
                bool free_ok = true;
                for (int st = s0; st < s0 + R && free_ok; ++st) {
                    const int j = last_use(st, nkb);
                    if (j >= 0) free_ok = wait_bounded(ptx::smem_u32(empty + st), (uint32_t)((j / S) & 1), abort_flag, wlim);
                }
                if (free_ok)
                    for (int r = 0; r < C; ++r)
                        if ((uint32_t)r != rank) ptx::mbar_arrive_remote(ptx::map_to_rank(ptx::smem_u32(freeb), (uint32_t)r));
            }
        }
        __syncwarp();
        if (C > 1) ptx::cluster_arrive();   // this warp is done with the cluster's shared memory
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        ptx::grid_dep_wait();
        if (lane == 0) {
            const uint32_t idesc = decode_idesc(KIND, BN);
            int stage = 0;
            uint32_t phase = 0;
            // FQ: the epilogue warps have written the token codes
            bool ok = !FQ || wait_bounded(ptx::smem_u32(a_ready), 0, abort_flag, wlim);
            for (int i = 0; i < nkb && ok; ++i) {
                ok = wait_bounded(ptx::smem_u32(full + stage), phase, abort_flag, wlim);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint64_t dA = FQ ? smem_desc(ptx::smem_u32(a_region + (size_t)i * m8 * 128))
                                       : smem_desc(ptx::smem_u32(a_slot(stage)));
                const uint64_t dW = smem_desc(ptx::smem_u32(w_slot(stage)));
#pragma unroll
                for (int k = 0; k < 4; ++k) {   // 32 K-bytes per MMA: +2 in 16-byte descriptor units
                    const uint32_t acc = (i == 0 && k == 0) ? 0u : 1u;
                    if (KIND == KIND_I8) ptx::mma_i8(tmem, dA + 2 * k, dW + 2 * k, idesc, acc);
                    else                 ptx::mma_f8f6f4(tmem, dA + 2 * k, dW + 2 * k, idesc, acc);
                }
                ptx::mma_commit(ptx::smem_u32(empty + stage));
                if (++stage == S) { stage = 0; phase ^= 1u; }
            }
            if (ok) {
                ptx::mma_commit(ptx::smem_u32(tfull));
            } else {
                // MMAs already issued finish before the tensor memory is released (bounded)
                ptx::mma_commit(ptx::smem_u32(drain));
                settle_local(ptx::smem_u32(drain), 0);
            }
        }
        __syncwarp();
        if (C > 1) ptx::cluster_arrive();   // this warp is done with the cluster's shared memory
    } else {
        // ------------------------------------------------------------ epilogue
        ptx::grid_dep_wait();
        const int q = warp & 3;                    // TMEM lane quadrant of this warp
        const int m = q * 16 + (lane & 15);        // token of this thread (lanes 16..31: none)
        const bool has_tok = lane < 16 && m < M;
        const bool warp_has_tok = q * 16 < M;
        const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
        const int te = threadIdx.x - 64;           // 0..127
        const bool dbg = a.out_i32 != nullptr;
        const int w = share((int)rank);            // columns this rank finishes
        const int cbase = n0 + (int)rank * SW;     // the first of them
        // their weight scales and the token scales: the loads go out now, while the MMAs
        // run, into registers (an HBM load issued behind the weight stream can take
        // microseconds; nothing waits for it before the accumulator is complete)
        float sw_r[2] = {0.0f, 0.0f}, sa_r = 0.0f;
        if (!dbg) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int c = te + j * kEpiThreads;
                if (c < w && cbase + c < a.N) sw_r[j] = __ldg(a.sW + cbase + c);
            }
            if (!FQ && te < M) sa_r = __ldg(a.sA + te);
        }
        if (FQ) {
            // ---- the activation quantizer, fused: per-token maxima over the row (this
            // rank's columns, then the other ranks' through distributed shared memory), the
            // scales, and the codes of this rank's K blocks written where the MMAs read them.
            // The same scale rule and quotient as the quantizer kernels, so the same codes.
            constexpr int QF = (KIND == KIND_I8) ? W8_Q_INT8 : W8_Q_FP8;
            constexpr int kB = 4;   // 16-value chunks per thread with their loads in flight together
            uint32_t* my_amax = amax_slots + rank * 64;
            if (te < 64) my_amax[te] = 0u;
            ptx::bar_sync(kEpiBarrier, kEpiThreads);
            const int kc0 = kb0 * 128;
            const int kc1 = min(a.K, (kb0 + nkb) * 128);
            const int nch = (kc1 - kc0) >> 4;   // 16-value chunks of a token row (K % 16 == 0)
            const int total = M * nch;          // chunk it: token it / nch, chunk it % nch
            // a thread's chunks it = te + 128 j; when they all fit in one batch they stay in
            // registers for the codes, else the codes pass loads them again (from L2)
            const bool one_batch = total <= kEpiThreads * kB;
            uint4 xv[2 * kB];
            auto load_batch = [&](int base) {
#pragma unroll
                for (int j = 0; j < kB; ++j) {
                    const int it = base + j * kEpiThreads;
                    if (it < total) {
                        const int mt = it / nch;
                        const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)mt * a.ldx + kc0 + (it - mt * nch) * 16);
                        xv[2 * j] = __ldg(src);
                        xv[2 * j + 1] = __ldg(src + 1);
                    }
                }
            };
            // the trip count is the same for the 32 lanes of a warp (the warp's first chunk
            // decides it): the shuffles below need every lane
            for (int wbase = te - lane; wbase < total; wbase += kEpiThreads * kB) {
                const int base = wbase + lane;
                load_batch(base);
#pragma unroll
                for (int j = 0; j < kB; ++j) {
                    const int it = base + j * kEpiThreads;
                    const int mt = it < total ? it / nch : -1;
                    float lo[8], hi[8];
                    unpack_bf16x8(xv[2 * j], lo);
                    unpack_bf16x8(xv[2 * j + 1], hi);
                    float mx = 0.0f;   // fmaxf ignores NaN, as the quantizer kernels' maxima do
                    if (mt >= 0)
#pragma unroll
                        for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fmaxf(fabsf(lo[i]), fabsf(hi[i])));
                    // one atomic per warp when the warp's 32 chunks belong to one token
                    const int mt0 = __shfl_sync(0xFFFFFFFFu, mt, 0);
                    if (__all_sync(0xFFFFFFFFu, mt == mt0)) {
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
                        if (lane == 0 && mt0 >= 0 && mx > 0.0f) atomicMax(my_amax + mt0, __float_as_uint(mx));
                    } else if (mt >= 0 && mx > 0.0f) {
                        atomicMax(my_amax + mt, __float_as_uint(mx));   // nonnegative: ordered as integers
                    }
                }
            }
            ptx::bar_sync(kEpiBarrier, kEpiThreads);
            bool fq_ok = true;
            if (C > 1) {
                // this rank's maxima to every other rank (into the same slot row there)
                const int pieces = m8 >> 2;
                if (te < (C - 1) * pieces) {
                    const int j = te / pieces, pc = te - j * pieces;
                    const uint32_t r = (uint32_t)(j < (int)rank ? j : j + 1);
                    const uint4 v = *reinterpret_cast<const uint4*>(my_amax + 4 * pc);
                    ptx::st_async_v4(ptx::map_to_rank(ptx::smem_u32(my_amax + 4 * pc), r), v.x, v.y, v.z, v.w,
                                     ptx::map_to_rank(ptx::smem_u32(amaxb), r));
                }
                fq_ok = wait_bounded<true>(ptx::smem_u32(amaxb), 0, abort_flag, wlim);
                if (ptx::bar_red_or(kEpiBarrier, kEpiThreads, !fq_ok)) fq_ok = false;
            }
            // row maxima, scales and divisors; the row maximum and the divisor's parts are
            // kept in shared memory once every thread has read the slots
            uint32_t row_mx = 0u;
            if (te < M) {
                for (int r = 0; r < C; ++r) row_mx = max(row_mx, amax_slots[r * 64 + te]);
                sa_r = scale_from_amax(__uint_as_float(row_mx), QF == W8_Q_FP8 ? kE4M3Max : kInt8Max, false);
                s_a[te] = sa_r;
                if (a.dbg_s != nullptr && tile == 0 && rank == 0) a.dbg_s[te] = sa_r;
            }
            ptx::bar_sync(kEpiBarrier, kEpiThreads);
            if (te < M) my_amax[te] = row_mx;
            ptx::bar_sync(kEpiBarrier, kEpiThreads);
            // codes of the real chunks
            auto encode16 = [&](int it, const uint4& v0, const uint4& v1) {
                const int mt = it / nch, c = it - mt * nch;
                const int k = kc0 + c * 16;
                float lo[8], hi[8];
                unpack_bf16x8(v0, lo);
                unpack_bf16x8(v1, hi);
                const RowDivisor d = make_divisor(s_a[mt], __uint_as_float(my_amax[mt]));
                const uint2 c0 = encode8<QF>(lo, d), c1 = encode8<QF>(hi, d);
                const uint4 codes = make_uint4(c0.x, c0.y, c1.x, c1.y);
                const int kbl = c >> 3, c16 = c & 7;
                *reinterpret_cast<uint4*>(a_region + (size_t)kbl * m8 * 128 + (size_t)mt * 128 +
                                          (size_t)((c16 ^ (mt & 7)) << 4)) = codes;
                if (a.dbg_q != nullptr && tile == 0) *reinterpret_cast<uint4*>(a.dbg_q + (size_t)mt * a.K + k) = codes;
            };
            if (fq_ok) {
                for (int base = te; base < total; base += kEpiThreads * kB) {
                    if (!one_batch) load_batch(base);
#pragma unroll
                    for (int j = 0; j < kB; ++j) {
                        const int it = base + j * kEpiThreads;
                        if (it < total) encode16(it, xv[2 * j], xv[2 * j + 1]);
                    }
                }
            }
            // zero codes where no real chunk lands: rows past M, and the columns past K of
            // the rank's last K block (as the zero-filled box of the two-kernel path)
            const int pad_rows = m8 - M;
            const int kpad = nkb * 8 - nch;   // 16-byte chunks past K in the last block
            for (int it = te; it < pad_rows * nkb * 8 + M * kpad; it += kEpiThreads) {
                int mt, c;
                if (it < pad_rows * nkb * 8) {
                    mt = M + it / (nkb * 8);
                    c = it - (mt - M) * nkb * 8;
                } else {
                    const int r2 = it - pad_rows * nkb * 8;
                    mt = r2 / kpad;
                    c = nch + (r2 - mt * kpad);
                }
                const int kbl = c >> 3, c16 = c & 7;
                *reinterpret_cast<uint4*>(a_region + (size_t)kbl * m8 * 128 + (size_t)mt * 128 +
                                          (size_t)((c16 ^ (mt & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
            }
            // the tensor core reads the region through the async proxy
            ptx::fence_proxy_async_smem();
            ptx::bar_sync(kEpiBarrier, kEpiThreads);
            if (te == 0) ptx::mbar_arrive(ptx::smem_u32(a_ready));
        }
        bool ok = wait_bounded(ptx::smem_u32(tfull), 0, abort_flag, wlim);
        if (ptx::bar_red_or(kEpiBarrier, kEpiThreads, !ok)) ok = false;
        ptx::tc_fence_after();
        const uint32_t recvb_s = ptx::smem_u32(recvb);
        // shared-memory address of every rank's receive area (the same layout in every
        // CTA of the cluster; the stage it starts at depends on the rank's K blocks)
        uint32_t* recv_at = reinterpret_cast<uint32_t*>(s_a + 64);   // [8]
        if (te < C) recv_at[te] = ptx::smem_u32(smem) + (uint32_t)(recv_stage(te) * stage_bytes);
        if (!dbg) {
#pragma unroll
            for (int j = 0; j < 2; ++j)
                if (te + j * kEpiThreads < w) s_w[te + j * kEpiThreads] = sw_r[j];
            if (te < M) s_a[te] = sa_r;
        }
        ptx::bar_sync(kEpiBarrier, kEpiThreads);
        // 4 accumulator words of token mt, columns [r SW + cc, r SW + cc + 4) of the tile,
        // to rank r, which finishes them ([source rank][token][column] in its receive area)
        auto deliver = [&](int mt, int r, int cc, uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3) {
            const int word = ((int)rank * M + mt) * RS + cc;
            if (r == (int)rank) {
                *reinterpret_cast<uint4*>(recv + word) = make_uint4(x0, x1, x2, x3);
            } else {
                ptx::st_async_v4(ptx::map_to_rank(recv_at[r], (uint32_t)r) + (uint32_t)word * 4u, x0, x1, x2, x3,
                                 ptx::map_to_rank(recvb_s, (uint32_t)r));
            }
        };
        auto wait_free = [&]() {
            // every other rank's receive area is free
            const bool f = wait_bounded<true>(ptx::smem_u32(freeb), 0, abort_flag, wlim);
            if (ptx::bar_red_or(kEpiBarrier, kEpiThreads, !f)) ok = false;
        };
        if (ok && use_stg) {
            // few tokens: the token lanes copy their rows out of tensor memory into the
            // staging area (while the other ranks may still be finishing), then all 128
            // threads send 16-byte pieces
            if (warp_has_tok) {
#pragma unroll 1
                for (int b = 0; b < BN; b += 64) {
                    uint32_t v[64];
                    ptx::tmem_ld64(t_lane + (uint32_t)b, v);
                    if (!has_tok) continue;
                    uint4* dst = reinterpret_cast<uint4*>(stg + m * BN + b);
#pragma unroll
                    for (int u = 0; u < 16; ++u)
                        if (b + 4 * u < BN) dst[u] = make_uint4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                }
            }
            ptx::bar_sync(kEpiBarrier, kEpiThreads);
            wait_free();
            if (ok) {
                const int q4 = BN >> 2;   // 16-byte pieces per token row
                for (int idx = te; idx < M * q4; idx += kEpiThreads) {
                    const int mt = idx / q4, c = 4 * (idx - mt * q4);
                    const uint4 x = *reinterpret_cast<const uint4*>(stg + mt * BN + c);
                    const int r = c / SW;
                    deliver(mt, r, c - r * SW, x.x, x.y, x.z, x.w);
                }
            }
        } else if (ok && C == 1) {
            // the whole K range is here: the token lanes copy their rows into the receive area
            if (warp_has_tok) {
#pragma unroll 1
                for (int b = 0; b < BN; b += 64) {
                    uint32_t v[64];
                    ptx::tmem_ld64(t_lane + (uint32_t)b, v);
                    if (!has_tok) continue;
                    uint4* dst = reinterpret_cast<uint4*>(recv + m * RS + b);
#pragma unroll
                    for (int u = 0; u < 16; ++u)
                        if (b + 4 * u < BN) dst[u] = make_uint4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                }
            }
        } else if (ok) {
            wait_free();
            if (ok && warp_has_tok) {
                // the token lanes read 64 accumulator columns per TMEM load and deliver them,
                // following the owning rank along the columns
#pragma unroll 1
                for (int b = 0; b < BN; b += 64) {
                    uint32_t v[64];
                    ptx::tmem_ld64(t_lane + (uint32_t)b, v);
                    if (!has_tok) continue;
                    int r = b / SW, cc = b - r * SW;
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        if (b + 4 * u < BN) deliver(m, r, cc, v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                        cc += 4;
                        if (cc == SW) { cc = 0; ++r; }
                    }
                }
            }
        }
        // this rank's own partials and the scales are in place; then the others' partials
        ptx::bar_sync(kEpiBarrier, kEpiThreads);
        if (ok && C > 1) {
            const bool g = wait_bounded<true>(ptx::smem_u32(recvb), 0, abort_flag, wlim);
            if (ptx::bar_red_or(kEpiBarrier, kEpiThreads, !g)) ok = false;
        }
        // every exchange with the other ranks is over (what this rank sent has landed in
        // theirs once they pass this point)
        if (C > 1) ptx::cluster_arrive();
        if (ok) {
            // add the C partials of every (token, column) of this rank's share in rank
            // order, scale and store: eight neighbouring columns per thread
            const int oct = w >> 3;
            for (int e = te; e < M * oct; e += kEpiThreads) {
                const int mm = e / oct;
                const int c = 8 * (e - mm * oct);
                const int n = cbase + c;
                if (n >= a.N) continue;
                uint32_t acc[8];
                {
                    const uint4* p = reinterpret_cast<const uint4*>(recv + mm * RS + c);
                    const uint4 x = p[0], y = p[1];
                    acc[0] = x.x; acc[1] = x.y; acc[2] = x.z; acc[3] = x.w;
                    acc[4] = y.x; acc[5] = y.y; acc[6] = y.z; acc[7] = y.w;
                }
                for (int r = 1; r < C; ++r) {
                    const uint4* p = reinterpret_cast<const uint4*>(recv + (r * M + mm) * RS + c);
                    const uint4 x = p[0], y = p[1];
                    acc[0] = add_words<KIND>(acc[0], x.x); acc[1] = add_words<KIND>(acc[1], x.y);
                    acc[2] = add_words<KIND>(acc[2], x.z); acc[3] = add_words<KIND>(acc[3], x.w);
                    acc[4] = add_words<KIND>(acc[4], y.x); acc[5] = add_words<KIND>(acc[5], y.y);
                    acc[6] = add_words<KIND>(acc[6], y.z); acc[7] = add_words<KIND>(acc[7], y.w);
                }
                const size_t o = (size_t)mm * a.N + n;
                const int nv = min(8, a.N - n);   // columns inside the output
                if (dbg) {
                    for (int j = 0; j < nv; ++j) a.out_i32[o + j] = (int32_t)acc[j];
                    continue;
                }
                const float sr = s_a[mm];
                float f[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) f[j] = __fmul_rn(__fmul_rn(word_to_float<KIND>(acc[j]), sr), s_w[c + j]);
                if (nv == 8 && a.vec_ok) {
                    *reinterpret_cast<uint4*>(a.out + o) =
                        make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                                   pack_bf16x2(f[6], f[7]));
                } else {
                    for (int j = 0; j < nv; ++j) a.out[o + j] = __float2bfloat16_rn(f[j]);
                }
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before();
    __syncthreads();
    // no rank leaves while another may still write into its shared memory or signal
    // its barriers (every thread of every rank arrived above, after its last exchange;
    // every wait there is bounded, so every rank gets there)
    if (C > 1) ptx::cluster_wait();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, tmem_cols);
    }
}

template <int KIND, bool FQ>
cudaError_t launch_kind(const GemmPlan& p, const GemmMaps& maps, const GemmArgs& args, cudaStream_t s)
{
    auto kern = gemm_decode_kernel<KIND, FQ>;
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
    if (p.split > 1) {
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

}  // namespace

cudaError_t launch_decode(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s)
{
    if (!p.decode || p.swap || p.G % p.split != 0) return cudaErrorNotSupported;
    if (p.fq)
        return p.fmt == W8_FMT_INT8 ? launch_kind<KIND_I8, true>(p, m, a, s) : launch_kind<KIND_F8, true>(p, m, a, s);
    return p.fmt == W8_FMT_INT8 ? launch_kind<KIND_I8, false>(p, m, a, s) : launch_kind<KIND_F8, false>(p, m, a, s);
}

int status_decode(int clear) { return status_word(clear); }

}  // namespace gemm
}  // namespace w8
