// w8_gemm_pair.cu -- the Standard full-K tile loop on CTA pairs (prefill sizes).
//
// Same arithmetic as the Standard form of gemm_kernel (FP8-dynamic and W8A8-INT8 scaled
// GEMM, [FP8] "Unified 8-bit GEMM" / [IT] third paragraph): out[m, n] = bf16(sA[m] sW[n]
// sum_k Aq[m, k] Wq[n, k]) with fp32 (int32) accumulation over the whole K range in one
// accumulator.  The output tile is 256 tokens x 256 weight rows, computed by a cluster
// of two CTAs on two SMs with one tcgen05 MMA of M = 256 (cta_group::2):
//   * each CTA loads, per 128-column K block, its own 128 token rows and 128 of the
//     tile's 256 weight rows (32 KB per stage instead of the 48 KB a one-CTA 128 x 256
//     tile needs), so the same shared memory holds five or six stages instead of four;
//   * both CTAs' loads signal the leader's (rank 0) full barrier, on which the leader
//     alone expects the bytes of both;
//   * the leader issues the MMAs; they read the A rows and the B rows of both CTAs at the
//     same shared-memory offsets and write each CTA's 128 accumulator rows into its own
//     tensor memory; the commits arrive on the stage and accumulator barriers of both;
//   * each CTA's epilogue scales and stores its own 128 token rows, then tells the
//     leader (remote arrive for rank 1) that the accumulator may be reused.
// Split-K (split S = 2..8, a power of two): pair p computes K chunk p % S (contiguous K
// blocks [c kbs / S, (c + 1) kbs / S)) of tile p / S, one unit per pair, so the grid has
// 2 tiles S CTAs (at most one per SM pair, all resident at once).  Each CTA publishes its
// 128 x 256 partial sums to its own workspace slot ([column][row] words) and counts itself
// in on its half-tile's counter; once all S are in, contributor c adds, for its slice of
// 256 / S columns, the S slots in chunk order -- a fixed order, so the result does not
// depend on timing -- then scales and stores; the last to leave resets the counters.  This fills the chip when a few tall tiles carry
// a long K (the down projection at a few hundred tokens: 16 tiles of K = 12288).
// Every wait is bounded (1 s, abort flag, device status W8_ERR_DEVICE_TIMEOUT).  No load
// uses cluster multicast.
#include "w8_gemm_kernel.cuh"

namespace w8 {
namespace gemm {
namespace {

constexpr int kHalfBytes = 128 * 128;          // one 128-row x 128-byte box
constexpr int kPairStage = 2 * kHalfBytes;     // per CTA: A half + B half of one K block
constexpr uint32_t kPairCols = 512;            // two 256-column fp32 / s32 accumulators

// ---- cta_group::2 forms of the tcgen05 / TMA instructions
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols)
{
    // one warp of each CTA of the pair, same warp index, same column count
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Load one box into this CTA's shared memory; the transaction bytes are counted on
// `bar` (a shared::cluster address, here the leader's barrier).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* tmap, uint32_t bar, int32_t x, int32_t y,
                                                 uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar), "l"(policy)
        : "memory");
}

template <int KIND>
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate)
{
    if (KIND == KIND_I8)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
            : "memory");
}

// Arrive on the barrier at this shared-memory offset in every CTA of `mask` once the
// pair MMAs issued so far have completed.
__device__ __forceinline__ void commit_pair(uint32_t bar, uint16_t mask)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                     bar),
                 "h"(mask)
                 : "memory");
}

// Bounded spin on a local barrier phase without touching the abort flag (unwinding).
__device__ __forceinline__ void settle(uint32_t bar, uint32_t parity)
{
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(bar, parity) && ptx::globaltimer_ns() - t0 < 10000000ull) {}
}

template <int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const GemmArgs a)
{
    constexpr uint32_t kIdesc = instr_desc<KIND, 256, 256>();
    extern __shared__ uint8_t smem_raw[];
    // the same offsets in both CTAs: the MMA reads the peer's operands at the leader's
    // addresses
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = a.stages;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * kPairStage);   // leader's are used
    uint64_t* empty = full + S;
    uint64_t* tfull = empty + S;
    uint64_t* tempty = tfull + 2;                                                   // leader's are used
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    auto a_slot = [&](int s) { return smem + (size_t)s * kPairStage; };
    auto b_slot = [&](int s) { return smem + (size_t)s * kPairStage + kHalfBytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();   // 0: the leader, which issues the MMAs

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(ptx::smem_u32(full + s), 1);
            ptx::mbar_init(ptx::smem_u32(empty + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(ptx::smem_u32(tfull + b), 1);
            ptx::mbar_init(ptx::smem_u32(tempty + b), 2 * kEpiThreads / 32);   // the epilogue warps of both CTAs
        }
        ptx::mbar_init(ptx::smem_u32(drain), 1);
        *abort_flag = 0;
        ptx::fence_barrier_init();
    }
    if (threadIdx.x == 32) {
        ptx::prefetch_tmap(&tmA);
        ptx::prefetch_tmap(&tmB);
    }
    __syncthreads();
    // both CTAs' barriers are initialised before either signals the other's
    ptx::cluster_sync();
    uint32_t tmem = 0;
    if (warp != 0) {
        if (warp == 1) {
            tmem_alloc_pair(ptx::smem_u32(tmem_slot), kPairCols);
            if (lane == 0) ptx::grid_dep_launch();
        }
        ptx::tc_fence_before();
        ptx::bar_sync(kTmemBarrier, kThreads - 32);
        ptx::tc_fence_after();
        tmem = *tmem_slot;
    }

    // pair p (the cluster) takes the tiles [p T / P, (p + 1) T / P), weight tile fastest
    // (token tile fastest, which reads each weight tile from HBM once, measured slower on
    // B200: 365 against 311 us at M = 4096, K = 4096, N = 24576); with a K split, the K
    // chunk p % S of tile p / S
    const int P = (int)(gridDim.x >> 1);
    const int pr = (int)(blockIdx.x >> 1);
    const int T = a.tiles;
    const int S_k = a.csplit > 1 ? a.csplit : 1;
    const int t0 = S_k > 1 ? pr / S_k : (int)((long long)pr * T / P);
    const int t1 = S_k > 1 ? t0 + 1 : (int)((long long)(pr + 1) * T / P);
    const int chunk = S_k > 1 ? pr % S_k : 0;
    const int kb0 = (int)((long long)chunk * a.kbs / S_k), kb1 = (int)((long long)(chunk + 1) * a.kbs / S_k);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_a = ptx::policy_evict_last();    // token rows: re-read by every weight tile
            const uint64_t pol_w = ptx::policy_evict_first();
            ptx::grid_dep_wait();
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int t = t0; t < t1 && ok; ++t) {
                const int rt = t / a.c_tiles, ct = t % a.c_tiles;
                const int ya = rt * 256 + (int)rank * 128, yb = ct * 256 + (int)rank * 128;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!wait_bounded(ptx::smem_u32(empty + stage), phase ^ 1u, abort_flag)) { ok = false; break; }
                    const uint32_t fb = ptx::map_to_rank(ptx::smem_u32(full + stage), 0);
                    if (rank == 0) ptx::mbar_arrive_expect_tx(ptx::smem_u32(full + stage), 2u * kPairStage);
                    tma_load_2d_pair(ptx::smem_u32(a_slot(stage)), &tmA, fb, kb * 128, ya, pol_a);
                    tma_load_2d_pair(ptx::smem_u32(b_slot(stage)), &tmB, fb, kb * 128, yb, pol_w);
                    ++issued;
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
            }
            if (ok) {
                // wait until the leader's MMAs have released every stage: the commits
                // arrive on this CTA's barriers asynchronously and must land before it
                // exits
                for (int j = 0; j < S; ++j) {
                    if (!wait_bounded(ptx::smem_u32(empty + stage), phase ^ 1u, abort_flag)) break;
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
            } else {
                // let this CTA's copies in flight land before it unwinds (bounded): the
                // leader sees them on its full barriers; the peer waits the same bound
                const long long lo = issued > S ? issued - S : 0;
                for (long long j = lo; j < issued; ++j) {
                    if (rank == 0) {
                        settle(ptx::smem_u32(full + (int)(j % S)), (uint32_t)((j / S) & 1));
                    } else {
                        const uint64_t tw = ptx::globaltimer_ns();
                        while (ptx::globaltimer_ns() - tw < 1000000ull) {}
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (rank == 0) {
            int stage = 0, buf = 0;
            uint32_t phase = 0, bphase = 0;
            bool ok = true;
            for (int t = t0; t < t1 && ok; ++t) {
                if (lane == 0) {
                    // both CTAs' epilogues have read this accumulator (the peer arrives remotely)
                    ok = wait_bounded<true>(ptx::smem_u32(tempty + buf), bphase ^ 1u, abort_flag);
                    ptx::tc_fence_after();
                    const uint32_t d_tmem = tmem + (uint32_t)(buf * 256);
                    for (int kb = kb0; kb < kb1 && ok; ++kb) {
                        ok = wait_bounded(ptx::smem_u32(full + stage), phase, abort_flag);
                        if (!ok) break;
                        ptx::tc_fence_after();
                        const uint64_t dA = smem_desc(ptx::smem_u32(a_slot(stage)));
                        const uint64_t dB = smem_desc(ptx::smem_u32(b_slot(stage)));
#pragma unroll
                        for (int k = 0; k < 4; ++k)   // 32 K-bytes per MMA: +2 in 16-byte units
                            mma_pair<KIND>(d_tmem, dA + 2 * k, dB + 2 * k, kIdesc, (kb == kb0 && k == 0) ? 0u : 1u);
                        commit_pair(ptx::smem_u32(empty + stage), 0x3);
                        if (++stage == S) { stage = 0; phase ^= 1u; }
                    }
                    if (ok) commit_pair(ptx::smem_u32(tfull + buf), 0x3);
                }
                ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
                if (++buf == 2) { buf = 0; bphase ^= 1u; }
            }
            if (!ok && lane == 0) {
                // MMAs already issued finish before the tensor memory is released (bounded)
                commit_pair(ptx::smem_u32(drain), 0x1);
                settle(ptx::smem_u32(drain), 0);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        ptx::grid_dep_wait();
        const int i = (warp & 3) * 32 + lane;   // accumulator row (TMEM lane) of this thread
        const int te = threadIdx.x - 64;        // 0 .. 127 over the epilogue warps
        const uint32_t t_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        constexpr size_t kSlotWords = 256 * 128;
        int buf = 0;
        uint32_t bphase = 0;
        for (int t = t0; t < t1; ++t) {
            const int rt = t / a.c_tiles, ct = t % a.c_tiles;
            const bool w = wait_bounded(ptx::smem_u32(tfull + buf), bphase, abort_flag);
            if (ptx::bar_red_or(kEpiBarrier, kEpiThreads, !w)) break;
            ptx::tc_fence_after();
            const int r_row = rt * 256 + (int)rank * 128 + i;   // token
            const bool has_row = r_row < a.M;
            const float s_row = (has_row && a.out_i32 == nullptr) ? __ldg(a.sA + r_row) : 1.0f;
            const int c_base = ct * 256;
            if (S_k == 1) {
#pragma unroll 1
                for (int c0 = 0; c0 < 256; c0 += 16) {
                    if (c_base + c0 >= a.N) break;
                    uint32_t v[16];
                    ptx::tmem_ld16(t_lane + (uint32_t)(buf * 256 + c0), v);
                    if (has_row) store_chunk16<KIND, false>(a, a.sA, r_row, c_base + c0, v, s_row);
                }
            } else {
                // publish this CTA's partial sums: [column][row] words, 512 contiguous bytes
                // per column over the 128 threads
                uint32_t* my = a.partials + ((size_t)pr * 2 + rank) * kSlotWords;
#pragma unroll 1
                for (int c0 = 0; c0 < 256; c0 += 16) {
                    if (c_base + c0 >= a.N) break;
                    uint32_t v[16];
                    ptx::tmem_ld16(t_lane + (uint32_t)(buf * 256 + c0), v);
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) __stcg(my + (size_t)(c0 + jj) * 128 + i, v[jj]);
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) ptx::mbar_arrive(ptx::smem_u32(tempty + buf));
                else ptx::mbar_arrive_remote(ptx::map_to_rank(ptx::smem_u32(tempty + buf), 0));
            }
            if (++buf == 2) { buf = 0; bphase ^= 1u; }
            if (S_k > 1) {
                // every contributor of the half-tile finishes a column slice once all S have
                // published (they are all resident: one unit per pair, at most one pair per
                // two SMs), adding the S partials in chunk order; the last to leave resets
                // the half-tile's two counters ([arrived, departed]) for the next call
                int* cnt = a.counters + ((size_t)t * 2 + rank) * 2;
                __threadfence();
                ptx::bar_sync(kEpiBarrier, kEpiThreads);
                bool all_in = true;
                if (te == 0) {
                    atomicAdd(cnt, 1);
                    all_in = wait_count(cnt, S_k, abort_flag);
                }
                if (!ptx::bar_red_or(kEpiBarrier, kEpiThreads, !all_in)) {
                    __threadfence();
                    const int cw = 256 / S_k;   // columns of each contributor's slice
                    const int cs = chunk * cw;
#pragma unroll 1
                    for (int c0 = cs; c0 < cs + cw; c0 += 16) {
                        if (c_base + c0 >= a.N) break;
                        uint32_t v[16];
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) v[jj] = 0u;
                        // the S chunks' partials in chunk order, four in flight together
#pragma unroll 1
                        for (int cb = 0; cb < S_k; cb += 4) {
                            uint32_t x[4][16];
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                if (cb + k < S_k) {
                                    const uint32_t* p = a.partials + ((size_t)(t * S_k + cb + k) * 2 + rank) * kSlotWords +
                                                        (size_t)c0 * 128 + i;
#pragma unroll
                                    for (int jj = 0; jj < 16; ++jj) x[k][jj] = __ldcg(p + (size_t)jj * 128);
                                }
                            }
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                if (cb + k < S_k)
#pragma unroll
                                    for (int jj = 0; jj < 16; ++jj)
                                        v[jj] = (cb + k == 0) ? x[k][jj] : add_words<KIND>(v[jj], x[k][jj]);
                        }
                        if (has_row) store_chunk16<KIND, false>(a, a.sA, r_row, c_base + c0, v, s_row);
                    }
                    ptx::bar_sync(kEpiBarrier, kEpiThreads);
                    if (te == 0 && atomicAdd(cnt + 1, 1) == S_k - 1) {
                        cnt[0] = 0;
                        cnt[1] = 0;
                    }
                }
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before();
    __syncthreads();
    // neither CTA leaves while the other may still signal its barriers or the MMAs may
    // still read its shared memory
    ptx::cluster_sync();
    if (warp == 1) {
        ptx::tc_fence_after();
        tmem_dealloc_pair(tmem, kPairCols);
    }
}

template <int KIND>
cudaError_t launch_kind(const GemmPlan& p, const GemmMaps& maps, const GemmArgs& args, cudaStream_t s)
{
    auto kern = gemm_pair_kernel<KIND>;
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
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 2;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kern, maps.R, maps.C, args);
}

}  // namespace

cudaError_t launch_pair(const GemmPlan& p, const GemmMaps& m, const GemmArgs& a, cudaStream_t s)
{
    if (p.G % 2 != 0 || p.bn != 256 || p.swap) return cudaErrorNotSupported;
    return p.fmt == W8_FMT_INT8 ? launch_kind<KIND_I8>(p, m, a, s) : launch_kind<KIND_F8>(p, m, a, s);
}

int status_pair(int clear) { return status_word(clear); }

}  // namespace gemm
}  // namespace w8
