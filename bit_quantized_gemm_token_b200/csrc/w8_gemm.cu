// w8_gemm.cu -- host side of the scaled 8-bit GEMM: tensor maps, planning of the
// variant (tiles, partition, pipeline depth, workspace) and dispatch to the kernel
// families (w8_gemm_f8.cu, w8_gemm_i8.cu, w8_gemm_block.cu, w8_gemm_bm64.cu,
// w8_gemm_fq.cu, w8_gemm_grouped.cu, and the CTA-pair loop of w8_gemm_pair.cu).  The
// kernel itself and what it computes are described in w8_gemm_kernel.cuh.
#include <algorithm>

#include "w8_gemm_kernel.cuh"

namespace w8 {
using namespace gemm;
namespace {

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

// bf16 activation rows [rows, cols] with row stride ld elements, boxes of 128 elements x
// box_rows rows, unswizzled; rows past the end read as zeros
bool make_tmap_x(CUtensorMap* m, const void* base, int rows, int cols, int ld, int box_rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

constexpr int tile_bn(int id) { return 16 << id; }

size_t stage_bytes(int bm, int bn, int kps) { return (size_t)kps * ((size_t)bm * 128 + (size_t)bn * 128); }

size_t smem_for(int bm, int bn, int kps, int stages)
{
    return 1024 + (size_t)stages * stage_bytes(bm, bn, kps) + (size_t)(2 * stages + 2 * kNumAcc + 5) * 8 + 16;
}

int default_stages(int bn, int kps)
{
    // decode tiles: three two-block stages (about 110 KB) so that a CTA of the next GEMM
    // fits beside one of the current GEMM on each SM
    if (kps == 2) return bn <= 32 ? 3 : 2;
    switch (bn) {
    case 16: return 10;
    case 32: return 9;
    case 64: return 8;
    case 128: return 6;
    default: return 4;
    }
}

}  // namespace

// ---------------------------------------------------------------- planning
// Shared-memory layout of the decode form for q's tile (bn, split, m8, M, kbs; a_region
// for the fused-quantization form, whose stages carry weights only): the stage count
// (`stages`, 0 = the default depth), the request padded so that no more CTAs share an SM
// than its tensor memory holds, and the receive area of the K-split reduction.
int decode_layout(GemmPlan* q, int stages, bool fq)
{
    const int bn = q->bn, C = q->split, M = q->M;
    const size_t stage = (size_t)((fq ? 0 : q->m8) + bn) * 128;
    // default depth: about 108 KB of stages and token codes, the most that still lets a CTA
    // of the next GEMM share the SM (bytes in flight per SM are what sets the streaming rate)
    if (stages == 0) {
        const long long room = 110592 - (long long)q->a_region;
        stages = (int)std::max<long long>(2, std::min<long long>(8, room / (long long)stage));
    }
    if (stages < 2) return W8_ERR_UNSUPPORTED;
    q->stages = stages;
    // token codes (fq), stages, barriers, TMEM slot and flag, then the scales of the columns
    // a rank finishes and of the tokens, the ranks' receive-area addresses, and (fq) the
    // ranks' partial token maxima
    q->smem_bytes = 1024 + q->a_region + (size_t)stages * stage + (size_t)(2 * stages + 4 + (fq ? 2 : 0)) * 8 + 16 +
                    (256 + 64 + 8) * 4 + (fq ? (size_t)8 * 64 * 4 : 0);
    // No more CTAs of this kernel may share an SM than its tensor memory holds: a CTA
    // waiting for columns another CTA of the same grid holds, while that one waits for
    // its cluster peers, would stall the grid.  Shared memory (228 KB per SM, 1 KB
    // reserved per CTA) bounds the CTAs per SM, so pad the request until it does.
    {
        const size_t cols = bn <= 32 ? 32 : bn <= 64 ? 64 : bn <= 128 ? 128 : 256;
        const size_t max_ctas = 512 / cols;
        while (233472 / (q->smem_bytes + 1024) > max_ctas) q->smem_bytes += 1024;
    }
    if (q->smem_bytes > 232448) return W8_ERR_UNSUPPORTED;
    // the partial sums of the columns a rank finishes sit over its stage memory: over the
    // R stages, for each of the two K-block counts a rank can hold, whose last use comes
    // earliest (stage s last holds K block s + S floor((n - 1 - s) / S) of n)
    const size_t recv = (size_t)C * M * (q->sw + 4) * 4;
    if (recv > (size_t)stages * stage) return W8_ERR_UNSUPPORTED;
    q->recv_R = (int)((recv + stage - 1) / stage);
    q->nkb_lo = q->kbs / C;
    for (int h = 0; h < 2; ++h) {
        const int n = q->nkb_lo + h;
        int best = 0x7FFFFFFF;
        q->recv_first[h] = 0;
        for (int c0 = 0; c0 + q->recv_R <= stages; ++c0) {
            int worst = -1;
            for (int st = c0; st < c0 + q->recv_R; ++st)
                worst = std::max(worst, st < n ? st + stages * ((n - 1 - st) / stages) : -1);
            if (worst < best) { best = worst; q->recv_first[h] = c0; }
        }
    }
    return W8_OK;
}

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
    int kps = (variant >> W8_V_KPS_SHIFT) & 0x3;
    int cps = (variant >> W8_V_CPS_SHIFT) & 0x3;
    q.pdl = (variant & W8_V_PDL) ? 1 : 0;
    q.cluster = (variant & W8_V_CLUSTER) ? 1 : 0;
    q.bm = (variant & W8_V_BM64) ? 64 : 128;
    q.pfix = (variant & W8_V_PFIX) ? 1 : 0;
    if (lg > 8) return W8_ERR_UNSUPPORTED;
    int rc_layout = W8_OK;
    if (variant & W8_V_DECODE) {
        // decode form (w8_gemm_decode.cu): tokens in the 64-row MMA operand, 16 (tile + 1)
        // weight rows in the wide one, split + 1 K chunks per weight tile as one cluster
        if (block || q.swap || q.stream || q.cluster || q.bm != 128 || q.pfix || (variant & W8_V_PAIR) || M > 64)
            return W8_ERR_UNSUPPORTED;
        const int bn = 16 * (tid + 1);
        const int C = lg + 1;
        if (bn < 64 || C > 8) return W8_ERR_UNSUPPORTED;
        q.kbs = (K + 127) / 128;
        if (C > q.kbs) return W8_ERR_UNSUPPORTED;
        q.decode = 1;
        q.bn = bn;
        q.split = C;
        q.kps = 1;
        q.m8 = (M + 7) & ~7;
        q.l2ahead = (variant >> W8_V_L2_SHIFT) & 0xF;
        q.sw = ((bn + 16 * C - 1) / (16 * C)) * 16;
        q.a_region = 0;
        rc_layout = decode_layout(&q, stages, false);
        if (rc_layout != W8_OK) return rc_layout;
        q.nsb = q.kbs;
        q.rows_R = M;
        q.rows_C = N;
        q.r_tiles = 1;
        q.c_tiles = (N + bn - 1) / bn;
        q.tiles = q.c_tiles;
        q.units = (long long)q.tiles * q.kbs;
        const long long g = (long long)q.tiles * C;
        if (g > 0x7FFFFFFF) return W8_ERR_UNSUPPORTED;
        q.G = (int)g;
        q.align_tiles = 1;
        q.ws_counters = 0;
        q.ws_bytes = 0;
        *p = q;
        return W8_OK;
    }
    if (variant & W8_V_PAIR) {
        // 256 x 256 tiles on CTA pairs: Standard full-K loop, FP8-dynamic / INT8; with a
        // K split, one (tile, K chunk) unit per pair
        if (block || q.swap || q.stream || lg > 3 || q.cluster || q.bm != 128 || q.pfix || tid != kTileBN256 ||
            kps > 1)
            return W8_ERR_UNSUPPORTED;
        if (stages == 0) stages = 5;   // measured: 5 a little ahead of 6 at M = 4096
        if (stages < 2) return W8_ERR_UNSUPPORTED;
        q.pair = 1;
        q.bn = 256;
        q.split = 1 << lg;
        q.kps = 1;
        q.stages = stages;
        q.kbs = (K + 127) / 128;
        q.nsb = q.kbs;
        if (q.split > q.kbs) return W8_ERR_UNSUPPORTED;
        q.smem_bytes = 1024 + (size_t)stages * 2 * 128 * 128 + (size_t)(2 * stages + 5) * 8 + 16;
        if (q.smem_bytes > 232448) return W8_ERR_UNSUPPORTED;
        q.rows_R = M;
        q.rows_C = N;
        q.r_tiles = (M + 255) / 256;
        q.c_tiles = (N + 255) / 256;
        q.tiles = q.r_tiles * q.c_tiles;
        q.units = (long long)q.tiles * q.nsb;
        const long long pairs_max = (sm_count > 0 ? sm_count : 148) / 2;
        if (q.split > 1) {
            // one unit per pair, every pair resident at once; a workspace slot of 128 x 256
            // words per CTA and two counters per half-tile
            const long long units = (long long)q.tiles * q.split;
            if (units > pairs_max || 4LL * q.tiles > kMaxCounterTiles) return W8_ERR_UNSUPPORTED;
            q.G = (int)(2 * units);
            q.align_tiles = 1;
            q.ws_counters = (size_t)kMaxCounterTiles * 4;
            q.ws_bytes = q.ws_counters + (size_t)units * 2 * 256 * 128 * 4;
            *p = q;
            return W8_OK;
        }
        const long long pairs = q.tiles < pairs_max ? q.tiles : pairs_max;
        if (pairs < 1) return W8_ERR_UNSUPPORTED;
        q.G = (int)(2 * pairs);
        q.align_tiles = 1;
        q.ws_counters = 0;
        q.ws_bytes = 0;
        *p = q;
        return W8_OK;
    }
    // the 64-row tile holds tokens: Standard form, FP8 / INT8, weight tiles of 128 or 256 rows
    if (q.bm == 64 && (q.swap || block || (tid != kTileBN128 && tid != kTileBN256))) return W8_ERR_UNSUPPORTED;
    // cluster split: 2, 4 or 8 K chunks, one cluster (portable size) per tile
    if (q.cluster && (q.stream || lg < 1 || lg > 3)) return W8_ERR_UNSUPPORTED;
    // the parallel fixup is written for the 64-row token tile's [row][column] partials
    if (q.pfix && (q.bm != 64 || q.cluster)) return W8_ERR_UNSUPPORTED;
    if (tid >= kNumTiles) return W8_ERR_UNSUPPORTED;
    q.bn = tile_bn(tid);
    if (block && q.bn > 64) return W8_ERR_UNSUPPORTED;   // block promotion keeps the tile in registers
    q.split = 1 << lg;
    q.kbs = (K + 127) / 128;
    if (kps == 3) return W8_ERR_UNSUPPORTED;
    if (kps == 0) {
        // two K blocks per stage for the narrow decode tiles (fewer, larger transfers per
        // stage), one for the wide tiles; one whenever the split needs the finer units
        kps = (q.bn <= 64) ? 2 : 1;
        if (!q.stream && q.split > (q.kbs + 1) / 2) kps = 1;
    }
    q.kps = kps;
    q.nsb = (q.kbs + kps - 1) / kps;
    if (stages == 0) stages = default_stages(q.bn, kps);
    if (stages < 2) return W8_ERR_UNSUPPORTED;
    q.stages = stages;
    q.smem_bytes = smem_for(q.bm, q.bn, kps, stages);
    // the cluster reduction reuses rank 0's stage memory for the partials: the other
    // ranks' [BN][BM] tiles, or, with the 64-row token tile, every rank's real rows
    if (q.cluster) {
        const size_t red = (q.bm == 64) ? (size_t)(1 << lg) * (size_t)(M < 64 ? M : 64) * q.bn * 4
                                        : (size_t)((1 << lg) - 1) * q.bn * q.bm * 4;
        if (red > (size_t)stages * stage_bytes(q.bm, q.bn, kps)) return W8_ERR_UNSUPPORTED;
    }
    if (q.smem_bytes > 232448) return W8_ERR_UNSUPPORTED;
    if (cps == 0) cps = 1;

    q.rows_R = q.swap ? N : M;
    q.rows_C = q.swap ? M : N;
    q.r_tiles = (q.rows_R + q.bm - 1) / q.bm;
    q.c_tiles = (q.rows_C + q.bn - 1) / q.bn;
    q.tiles = q.r_tiles * q.c_tiles;
    q.units = (long long)q.tiles * q.nsb;
    const long long sms = sm_count > 0 ? sm_count : 148;
    if (q.stream) {
        long long g = sms * cps;
        if (g > q.units) g = q.units;
        q.G = (int)g;
        q.align_tiles = 0;
    } else if (q.split > 1) {
        if (q.split > q.nsb) return W8_ERR_UNSUPPORTED;
        const long long g = (long long)q.tiles * q.split;
        if (g > 0x7FFFFFFF) return W8_ERR_UNSUPPORTED;
        q.G = (int)g;
        q.align_tiles = 0;
    } else {
        long long g = sms * cps;
        if (g > q.tiles) g = q.tiles;
        q.G = (int)g;
        q.align_tiles = 1;
    }
    // contributors of a tile wait for one another only if all CTAs can be resident at once
    if (q.pfix && q.G > sms) return W8_ERR_UNSUPPORTED;
    // partial slots exist whenever some tile's K range can be split across CTAs (the
    // cluster split reduces through distributed shared memory instead)
    const bool partials = !q.align_tiles && !(q.G == q.tiles) && !q.cluster;   // G == tiles: one whole tile per CTA
    if (partials) {
        // The counter area has one fixed size for every shape, so that the partial
        // slots of one call never lie where another call's counters are.
        if (q.tiles > kMaxCounterTiles) return W8_ERR_UNSUPPORTED;
        q.ws_counters = (size_t)kMaxCounterTiles * 4;
        q.ws_bytes = q.ws_counters + (size_t)q.G * 2 * (size_t)q.bn * q.bm * 4;
    } else {
        q.ws_counters = 0;
        q.ws_bytes = 0;
    }
    *p = q;
    return W8_OK;
}

// ---------------------------------------------------------------- launch
namespace {
// Arguments of the decode-form kernel (plain, or with the quantization fused: then the
// caller adds x and the debug outputs)
GemmArgs decode_args(const GemmPlan& p, const float* A_scale, const float* W_scale, void* out, int32_t* out_i32,
                     int starve, unsigned long long wait_ns)
{
    GemmArgs args = {};
    args.M = p.M; args.N = p.N; args.K = p.K;
    args.rows_R = p.M; args.rows_C = p.N;
    args.r_tiles = 1; args.c_tiles = p.c_tiles; args.tiles = p.tiles;
    args.kbs = p.kbs;
    args.nsb = p.kbs;
    args.units = p.units;
    args.G = p.G;
    args.align_tiles = 1;
    args.csplit = p.split;
    args.stages = p.stages;
    args.pdl = p.pdl;
    args.vec_ok = (p.N % 8 == 0) && ((reinterpret_cast<uintptr_t>(out) & 15) == 0);
    args.sA = A_scale;
    args.sW = W_scale;
    args.out = static_cast<__nv_bfloat16*>(out);
    args.out_i32 = out_i32;
    args.bn = p.bn;
    args.m8 = p.m8;
    args.l2ahead = p.l2ahead;
    args.sw = p.sw;
    args.recv_R = p.recv_R;
    args.nkb_lo = p.nkb_lo;
    args.recv_first[0] = p.recv_first[0];
    args.recv_first[1] = p.recv_first[1];
    args.a_region = (int)p.a_region;
    args.starve = starve;
    args.wait_ns = wait_ns;
    return args;
}
}  // namespace

int gemm_launch(const GemmPlan& p, const void* A_q, const float* A_scale, const void* W_q, const float* W_scale,
                void* out, int32_t* out_i32, void* workspace, size_t ws_bytes, cudaStream_t s, const int* g_off,
                int starve, unsigned long long wait_ns)
{
    if (p.ws_bytes > 0 && (workspace == nullptr || ws_bytes < p.ws_bytes)) return W8_ERR_WORKSPACE;
    if (p.ws_bytes > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255)) return W8_ERR_ALIGNMENT;
    if (p.decode) {
        // token box of M rounded up to 8 rows, weight box of bn rows
        GemmMaps maps;
        if (!make_tmap(&maps.R, A_q, p.M, p.K, p.m8)) return W8_ERR_CUDA;
        if (!make_tmap(&maps.C, W_q, p.N, p.K, p.bn)) return W8_ERR_CUDA;
        const GemmArgs args = decode_args(p, A_scale, W_scale, out, out_i32, starve, wait_ns);
        const cudaError_t e = launch_decode(p, maps, args, s);
        if (e == cudaErrorNotSupported) return W8_ERR_UNSUPPORTED;
        return e == cudaSuccess ? W8_OK : W8_ERR_CUDA;
    }
    CUtensorMap tR, tC;
    const void* R = p.swap ? W_q : A_q;
    const void* C = p.swap ? A_q : W_q;
    // the grouped form's weights are the experts' [N, K] matrices one after another
    if (!make_tmap(&tR, R, p.grouped ? p.rows_R * p.g_E : p.rows_R, p.K, p.bm)) return W8_ERR_CUDA;
    // a CTA of a pair loads half of the 256 weight rows of a tile
    if (!make_tmap(&tC, C, p.rows_C, p.K, p.pair ? 128 : p.bn)) return W8_ERR_CUDA;

    GemmArgs args = {};
    args.M = p.M; args.N = p.N; args.K = p.K;
    args.swap = p.swap;
    args.rows_R = p.rows_R; args.rows_C = p.rows_C;
    args.r_tiles = p.r_tiles; args.c_tiles = p.c_tiles; args.tiles = p.tiles;
    args.kbs = p.kbs;
    args.nsb = p.nsb;
    args.units = p.units;
    args.G = p.G;
    args.align_tiles = p.align_tiles;
    args.csplit = (p.cluster || p.pair) ? p.split : 0;
    args.pfix = p.pfix;
    args.grouped = p.grouped;
    args.g_E = p.g_E;
    args.g_off = g_off;
    args.w_ptr = static_cast<const uint8_t*>(W_q);
    args.stages = p.stages;
    args.pdl = p.pdl;
    args.ld_sblk = p.kbs;
    args.vec_ok = (p.N % 8 == 0) && ((reinterpret_cast<uintptr_t>(out) & 15) == 0);
    args.sA = A_scale;
    args.sW = W_scale;
    args.out = static_cast<__nv_bfloat16*>(out);
    args.out_i32 = out_i32;
    args.counters = p.ws_bytes ? static_cast<int*>(workspace) : nullptr;
    args.partials = p.ws_bytes ? reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + p.ws_counters) : nullptr;

    GemmMaps maps;
    maps.R = tR;
    maps.C = tC;
    cudaError_t e = cudaErrorInvalidValue;
    if (p.grouped)                 e = launch_grouped(p, maps, args, s);
    else if (p.pair)               e = launch_pair(p, maps, args, s);
    else if (p.fmt >= W8_FMT_BLOCK_FP8) e = launch_block(p, maps, args, s);
    else if (p.bm == 64)           e = launch_bm64(p, maps, args, s);
    else if (p.fmt == W8_FMT_INT8) e = launch_i8(p, maps, args, s);
    else                           e = launch_f8(p, maps, args, s);
    if (e == cudaErrorNotSupported) return W8_ERR_UNSUPPORTED;
    return e == cudaSuccess ? W8_OK : W8_ERR_CUDA;
}

// ---------------------------------------------------------------- fused quantize + GEMM
namespace {
long long host_unit_begin(const GemmPlan& q, long long g)
{
    if (q.align_tiles) return (g * q.tiles / q.G) * q.nsb;
    return g * q.units / q.G;
}
}  // namespace

int linear_plan(int fmt, int M, int N, int K, int variant, int sm_count, GemmPlan* p)
{
    GemmPlan q;
    int rc = gemm_plan(fmt, M, N, K, variant, sm_count, &q);
    if (rc != W8_OK) return rc;
    if (q.decode) {
        // decode form: the codes of the rank's K blocks for every token, in a region ahead
        // of stages that carry weights only (the 64-row MMA reads past the last block's
        // rows into the stages: rows that are never stored)
        const int nkb_max = (q.kbs + q.split - 1) / q.split;
        q.a_region = ((size_t)nkb_max * q.m8 * 128 + 1023) & ~(size_t)1023;
        // the variant's stage count, or fewer if the code region needs the room
        int st = (variant >> W8_V_STAGES_SHIFT) & 0xF;
        rc = decode_layout(&q, st, true);
        while (rc != W8_OK && st > 2) rc = decode_layout(&q, --st, true);
        if (rc != W8_OK) return rc;
        q.fq = 1;
        *p = q;
        return W8_OK;
    }
    // the activations are the narrow C operand of a Swap-AB tile holding every token
    if (!q.swap || q.bm != 128 || q.pfix || q.c_tiles != 1 || q.bn > 64) return W8_ERR_UNSUPPORTED;
    int rg = 0;
    for (long long g = 0; g < q.G; ++g) {
        int lo = 0, n = 0;
        region_of(host_unit_begin(q, g), host_unit_begin(q, g + 1), q.nsb, q.kps, q.kbs, &lo, &n);
        if (n > rg) rg = n;
    }
    // x is staged by TMA: the region's K blocks, or whole rows when per-token maxima are
    // taken without a cluster split (then every CTA reads its rows in full)
    const int m8 = (M + 7) & ~7;
    const bool full_rows = fmt < W8_FMT_BLOCK_FP8 && !q.cluster;
    const int xkb = full_rows ? q.kbs : rg;
    // the stages carry weights only; fewer of them if the region needs the room
    int st = q.stages;
    while (st > 2 && fq_smem_bytes(q.bn, q.kps, st, rg, m8, xkb) > 232448) --st;
    if (fq_smem_bytes(q.bn, q.kps, st, rg, m8, xkb) > 232448) return W8_ERR_UNSUPPORTED;
    if (q.cluster && (size_t)(q.split - 1) * q.bn * q.bm * 4 > (size_t)st * q.kps * q.bm * 128) return W8_ERR_UNSUPPORTED;
    q.stages = st;
    q.rg_max_kb = rg;
    q.fq_m8 = m8;
    q.fq_xkb = xkb;
    q.fq_full_rows = full_rows ? 1 : 0;
    q.smem_bytes = fq_smem_bytes(q.bn, q.kps, st, rg, m8, xkb);
    q.fq = 1;
    *p = q;
    return W8_OK;
}

int grouped_plan(int fmt, int T, int N, int K, int E, int max_m, int variant, int sm_count, GemmPlan* p)
{
    if (E <= 0 || max_m <= 0 || max_m > T) return W8_ERR_INVALID_ARG;
    if (fmt != W8_FMT_FP8_DYN && fmt != W8_FMT_INT8) return W8_ERR_UNSUPPORTED;
    GemmPlan q;
    // the shape of one expert's GEMM at its largest token count fixes the tiles
    int rc = gemm_plan(fmt, max_m, N, K, variant, sm_count, &q);
    if (rc != W8_OK) return rc;
    // Swap-AB, balanced partition over the SMs, reductions through the workspace
    if (!q.swap || !q.stream || q.cluster || q.pfix || q.bm != 128) return W8_ERR_UNSUPPORTED;
    const long long tiles_max = (long long)E * q.r_tiles * q.c_tiles;
    if (tiles_max > kMaxCounterTiles) return W8_ERR_UNSUPPORTED;
    q.grouped = 1;
    q.g_E = E;
    q.M = T;
    q.rows_C = T;
    // one CTA per SM (or the variant's CTAs per SM): the units are counted on the device
    const int cps = ((variant >> W8_V_CPS_SHIFT) & 0x3) ? ((variant >> W8_V_CPS_SHIFT) & 0x3) : 1;
    q.G = (sm_count > 0 ? sm_count : 148) * cps;
    // tile counts and offsets of the experts, kept in shared memory
    q.smem_bytes += (size_t)(2 * (E + 1)) * 4 + 16;
    if (q.smem_bytes > 232448) return W8_ERR_UNSUPPORTED;
    // the balanced partition deals out the units of the experts that have tokens; the
    // partial slots are per CTA and the counter area has its fixed size
    q.ws_counters = (size_t)kMaxCounterTiles * 4;
    q.ws_bytes = q.ws_counters + (size_t)q.G * 2 * (size_t)q.bn * q.bm * 4;
    *p = q;
    return W8_OK;
}

int linear_launch(const GemmPlan& p, const void* x, int ldx, const void* W_q, const float* W_scale, void* out,
                  void* workspace, size_t ws_bytes, uint8_t* dbg_q, float* dbg_s, cudaStream_t s)
{
    if (!p.fq) return W8_ERR_INVALID_ARG;
    if (p.ws_bytes > 0 && (workspace == nullptr || ws_bytes < p.ws_bytes)) return W8_ERR_WORKSPACE;
    if (p.ws_bytes > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255)) return W8_ERR_ALIGNMENT;
    if (p.decode) {
        // weight boxes only: the kernel reads x and writes the token codes itself
        GemmMaps maps;
        if (!make_tmap(&maps.C, W_q, p.N, p.K, p.bn)) return W8_ERR_CUDA;
        maps.R = maps.C;
        GemmArgs args = decode_args(p, nullptr, W_scale, out, nullptr, 0, 0);
        args.x = static_cast<const __nv_bfloat16*>(x);
        args.ldx = ldx;
        args.dbg_q = dbg_q;
        args.dbg_s = dbg_s;
        const cudaError_t e = launch_decode(p, maps, args, s);
        if (e == cudaErrorNotSupported) return W8_ERR_UNSUPPORTED;
        return e == cudaSuccess ? W8_OK : W8_ERR_CUDA;
    }
    CUtensorMap tR, tX;
    if (!make_tmap(&tR, W_q, p.rows_R, p.K, p.bm)) return W8_ERR_CUDA;
    if (!make_tmap_x(&tX, x, p.M, p.K, ldx, p.fq_m8)) return W8_ERR_CUDA;
    GemmArgs args = {};
    args.M = p.M; args.N = p.N; args.K = p.K;
    args.swap = p.swap;
    args.rows_R = p.rows_R; args.rows_C = p.rows_C;
    args.r_tiles = p.r_tiles; args.c_tiles = p.c_tiles; args.tiles = p.tiles;
    args.kbs = p.kbs;
    args.nsb = p.nsb;
    args.units = p.units;
    args.G = p.G;
    args.align_tiles = p.align_tiles;
    args.csplit = (p.cluster || p.pair) ? p.split : 0;
    args.w_ptr = static_cast<const uint8_t*>(W_q);
    args.stages = p.stages;
    args.pdl = p.pdl;
    args.ld_sblk = p.kbs;
    args.vec_ok = 0;
    args.sA = nullptr;
    args.sW = W_scale;
    args.out = static_cast<__nv_bfloat16*>(out);
    args.out_i32 = nullptr;
    args.counters = p.ws_bytes ? static_cast<int*>(workspace) : nullptr;
    args.partials = p.ws_bytes ? reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + p.ws_counters) : nullptr;
    args.x = static_cast<const __nv_bfloat16*>(x);
    args.ldx = ldx;
    args.fq_block = p.fmt >= W8_FMT_BLOCK_FP8;
    args.fq_ue8m0 = p.fmt == W8_FMT_BLOCK_FP8_UE8M0;
    args.rg_max_kb = p.rg_max_kb;
    args.fq_m8 = p.fq_m8;
    args.fq_xkb = p.fq_xkb;
    args.fq_full_rows = p.fq_full_rows;
    args.dbg_q = dbg_q;
    args.dbg_s = dbg_s;
    GemmMaps maps;
    maps.R = tR;
    maps.C = tX;   // the bf16 activation rows, staged for the in-kernel quantization
    const cudaError_t e = launch_fq(p, maps, args, s);
    if (e == cudaErrorNotSupported) return W8_ERR_UNSUPPORTED;
    return e == cudaSuccess ? W8_OK : W8_ERR_CUDA;
}

// CTAs of the plan's kernel that fit on one SM together (registers, shared memory,
// threads): 2 means a CTA of this GEMM can sit beside one of the same size.
int gemm_occupancy(const GemmPlan& p, int* n)
{
    GemmMaps maps = {};
    maps.occupancy = n;
    GemmArgs args = {};
    cudaError_t e = cudaErrorInvalidValue;
    if (p.decode)                  e = launch_decode(p, maps, args, nullptr);
    else if (p.fq)                 e = launch_fq(p, maps, args, nullptr);
    else if (p.grouped)            e = launch_grouped(p, maps, args, nullptr);
    else if (p.pair)               e = launch_pair(p, maps, args, nullptr);
    else if (p.fmt >= W8_FMT_BLOCK_FP8) e = launch_block(p, maps, args, nullptr);
    else if (p.bm == 64)           e = launch_bm64(p, maps, args, nullptr);
    else if (p.fmt == W8_FMT_INT8) e = launch_i8(p, maps, args, nullptr);
    else                           e = launch_f8(p, maps, args, nullptr);
    if (e == cudaErrorNotSupported) return W8_ERR_UNSUPPORTED;
    return e == cudaSuccess ? W8_OK : W8_ERR_CUDA;
}

// First nonzero device status word over the kernel families (each unit has its own).
int gemm_device_status(int clear)
{
    int first = 0;
    for (int (*f)(int) : {status_f8, status_i8, status_block, status_bm64, status_fq, status_grouped, status_pair,
                          status_decode}) {
        const int v = f(clear);
        if (v == W8_ERR_CUDA) return v;
        if (v != 0 && first == 0) first = v;
    }
    return first;
}

}  // namespace w8
