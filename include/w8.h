/*
 * w8.h -- C ABI of libw8, the B200 (sm_100a) 8-bit quantized linear layer.
 *
 * The layer is a dynamic activation quantizer (or a fused rms_norm / silu_and_mul
 * producer) feeding one scaled GEMM that covers the Standard, Split-K and Swap-AB
 * variants in three 8-bit formats: FP8-dynamic, W8A8-INT8 and Block-FP8.  Sources
 * (web pages; no formulas are printed there, so each entry point states the
 * definition it computes):
 *   [FP8] "PyTorch integra Helion en vLLM para acelerar inferencia FP8"
 *         (noticias.mechatronicstore.cl) -- sections "Patron de fusion del forward
 *         pass" (rms_norm + fp8_quant, silu_and_mul + fp8_quant, scaled_mm as the
 *         linear op) and "Kernels Helion implementados" (the kernel list);
 *   [LIN] "Helion DSL added to vLLM to autotune linear inference backends"
 *         (signaltitans.com) -- "Unified GEMM Architecture" (one GEMM, Split-K and
 *         Swap-AB as parameters, FP8 Dynamic / W8A8 INT8 / Block FP8) and "Hybrid
 *         Dispatch and Autotuning" (small token counts under CUDA-graph replay);
 *   [IT]  "Helion nel backend vLLM: un solo GEMM, tuning per forma e guadagni fino
 *         al 10%" (ai-radar.it) -- paragraphs 2-4 (Split-K, Swap-AB as (B^T A^T)^T,
 *         split_k a power of two up to 256, per-shape configs).
 *
 * Conventions shared by every entry point
 *   - Tensors are DEVICE memory owned by the caller; the library never allocates
 *     device memory on these paths and never synchronises: every call only enqueues
 *     work on `stream` (NULL = the legacy default stream) and returns.
 *   - Layouts are row-major.  M = tokens, K = in-features, N = out-features.
 *     Activations x are bf16 [M, K] with row stride ldx (elements).  Codes are one byte
 *     each: e4m3 ("fn": max 448, no inf) or int8 in [-127, 127].  Weights are
 *     W[N, K] (K contiguous; the nn.Linear [out, in] layout).  GEMM output is bf16
 *     [M, N].  Scales are fp32.
 *   - Every call returns W8_OK (0) or a negative W8_ERR_* code; on an error nothing
 *     was enqueued.  No call aborts the process or traps on the device.
 *   - Quantization: s = amax / Q with Q = 448 (e4m3) or 127 (int8), an IEEE fp32
 *     division; codes = RNE(x / s) (true division), e4m3 saturating to +-448, int8
 *     clamped to [-127, 127].  An all-zero row or group gets s = 1 (codes 0).
 *     UE8M0 scales are s = 2^ceil(log2(amax/448)) (fp32 quotient), exponent clamped to
 *     [-127, 127]; they are still passed as fp32 values.
 *   - Input values are expected to be finite.
 */
#ifndef W8_H
#define W8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* w8_stream_t; /* identical to cudaStream_t */

#if defined(__GNUC__)
#define W8_API __attribute__((visibility("default")))
#else
#define W8_API
#endif

/* ---- status codes ---------------------------------------------------------- */
#define W8_OK 0
#define W8_ERR_INVALID_ARG (-1)     /* null pointer, non-positive size, bad enum     */
#define W8_ERR_UNSUPPORTED (-2)     /* format / variant / size not available          */
#define W8_ERR_ALIGNMENT (-3)       /* pointer or stride not aligned as required      */
#define W8_ERR_WORKSPACE (-4)       /* workspace missing or smaller than required     */
#define W8_ERR_CUDA (-5)            /* a CUDA runtime call (e.g. the launch) failed   */
#define W8_ERR_DEVICE_TIMEOUT (-6)  /* a bounded device-side wait gave up             */
#define W8_ERR_NO_DEVICE (-7)       /* current device is not an sm_100 (B200) part    */
#define W8_ERR_IO (-8)              /* table file missing or malformed                */

/* ---- activation quantizer formats ------------------------------------------ */
#define W8_Q_FP8 0
#define W8_Q_INT8 1

/* ---- GEMM formats -------------------------------------------------------------- */
#define W8_FMT_FP8_DYN 0          /* per-token sA[M] x per-channel sW[N]                  */
#define W8_FMT_INT8 1             /* same scales, int8 x int8 -> int32 accumulation       */
#define W8_FMT_BLOCK_FP8 2        /* sA[M, K/128] (1x128 groups), sW[N/128, K/128] blocks */
#define W8_FMT_BLOCK_FP8_UE8M0 3  /* as BLOCK_FP8, every scale an exact power of two      */

/* ---- GEMM variant word -----------------------------------------------------------
 * 0 (W8_VARIANT_AUTO) lets the library choose from its per-shape table (loaded with
 * w8_load_table) or, when the shape is not in it, from a built-in rule: up to 64 tokens
 * the decode form (W8_V_DECODE, tile and K chunks by a cost model) for FP8-dynamic and
 * INT8, Swap-AB with the balanced partition and a token tile of 16 / 32 / 64 for
 * Block-FP8; past 64 tokens W8_V_PAIR tiles for FP8-dynamic and INT8, and the 64-wide
 * balanced Standard loop for Block-FP8.  An explicit
 * variant sets W8_V_EXPLICIT plus:
 *   W8_V_SWAP_AB  compute out^T = W . Aq^T: the 128-row MMA slot runs over N and the
 *                 narrow slot over tokens (the Swap-AB variant, for small M);
 *                 otherwise the 128-row slot runs over tokens (Standard).
 *   split         log2 of split_k in bits 4..7 (split_k = 1..256, a power of two,
 *                 <= the tile's stage blocks): every output tile's K range is cut into split_k
 *                 chunks, one CTA each, and the fp32 (int32 for INT8) partials are
 *                 added in a fixed order (Split-K).  split = 0 without W8_V_STREAM is
 *                 the Standard full-K tile loop.
 *   W8_V_STREAM   balanced partition: the (tile, 128-column K block) units are dealt
 *                 out evenly to one CTA per SM, so a tile's K range may be split across
 *                 neighbouring CTAs (a Split-K whose chunk boundaries follow the SM
 *                 count); split bits are ignored.
 *   tile          bits 8..11, the narrow tile side BN: 0:16 1:32 2:64 3:128 4:256.
 *   stages        bits 12..15, shared-memory pipeline depth (0 = default).
 *   W8_V_CLUSTER  Split-K whose split_k (2, 4 or 8) chunks of a tile run as one
 *                 thread-block cluster: the partial accumulators are added in rank 0's
 *                 shared memory through distributed shared memory (no workspace).
 *   W8_V_BM64     Standard form with a 64-row token tile in the MMA's M slot and the
 *                 weights in its N slot (tile 128 or 256; FP8 / INT8).  Each MMA then
 *                 consumes BN weight rows; for decode sizes this carries twice the weight
 *                 bytes per tensor-core instruction of the 128-row Swap-AB tile.
 *   W8_V_PFIX     with W8_V_BM64 and without W8_V_CLUSTER: a tile whose K range is
 *                 shared by several CTAs is finished by all of them together.  Each one
 *                 publishes its partial, waits (bounded) until every contributor of the
 *                 tile has, then adds the contributors' partials in CTA order for its own
 *                 slice of the tile's columns.  This needs every CTA of the launch resident
 *                 at once (as a cooperative launch does), so the launch may not exceed the
 *                 SM count (ctas/SM must be 1).  Without it the contributor that arrives
 *                 last adds the whole tile alone.
 *   kps           bits 20..21, 128-column K blocks carried by one pipeline stage (0 =
 *                 default: 2 for BN <= 64, else 1).  The partition unit is one stage
 *                 block, so split_k must not exceed ceil(K / (128 * kps)).
 *   ctas/SM       bits 22..23, CTAs per SM for W8_V_STREAM and the Standard loop
 *                 (0 = 1).
 *   W8_V_PAIR     Standard tile loop (tile 256, no W8_V_STREAM / W8_V_CLUSTER /
 *                 W8_V_BM64; FP8-dynamic or INT8) over 256-token x 256-weight-row tiles,
 *                 each computed by a cluster of two CTAs on two SMs with one 256-row
 *                 tensor-core MMA (cta_group::2).  Each CTA loads 128 token rows and 128
 *                 weight rows per K block, and its tensor memory holds its 128 output
 *                 rows.  split field 0: the pairs take whole tiles in contiguous runs, one
 *                 accumulator over the whole K range, K blocks in order (the one-CTA
 *                 Standard loop's sum), no workspace.  split = 2, 4 or 8: one (tile, K
 *                 chunk) unit per pair -- legal only while tiles x split <= SMs / 2 and
 *                 split <= ceil(K / 128) -- each CTA's partial sums go to a workspace
 *                 slot; once all contributors of a half-tile have published, each adds
 *                 the split partials of its slice of columns in chunk order (a fixed
 *                 order), scales and stores; workspace as for the split partitions
 *                 (256 KiB of counters, then 256 KiB per unit).  Stages default to 5.  INT8 accumulators are exact either way.
 *                 With PDL the kernel waits for the kernels ahead before its first load.
 *   W8_V_DECODE   decode form (M <= 64; FP8-dynamic or INT8; no W8_V_SWAP_AB / W8_V_STREAM /
 *                 W8_V_CLUSTER / W8_V_BM64 / W8_V_PAIR): the tokens occupy the tensor
 *                 core's 64-row operand and BN = 16 * (tile + 1) weight rows (64..256) its
 *                 wide one, so each MMA consumes BN x 32 weight bytes.  The split field
 *                 holds C - 1: each weight tile's K range is cut into C = 1..8 contiguous
 *                 chunks (at most one per 128-column K block), run as one thread-block
 *                 cluster of C CTAs; their fp32 (int32 for INT8) partial sums are added in
 *                 chunk order in distributed shared memory, each rank finishing a share of
 *                 the tile's columns.  No workspace.  Stages as above (default 3); bits
 *                 27..30: K blocks of weights each CTA keeps in flight into L2 ahead of its
 *                 stages (0 = none).  The variant for decode token counts.
 *   W8_V_PDL      launch with programmatic dependent launch: the kernel may start while
 *                 earlier kernels on the stream still run, and it reads weight tiles
 *                 (into shared memory and L2) before waiting for them.  Only legal when
 *                 W_q was not written by work still in flight on the stream -- the
 *                 normal case of weights quantized once at load time.  Activations,
 *                 scales, outputs and workspace are touched only after the wait.
 */
#define W8_VARIANT_AUTO 0
#define W8_V_EXPLICIT (1 << 0)
#define W8_V_SWAP_AB (1 << 1)
#define W8_V_STREAM (1 << 2)
#define W8_V_SPLIT_SHIFT 4
#define W8_V_TILE_SHIFT 8
#define W8_V_STAGES_SHIFT 12
#define W8_V_PDL (1 << 16)
#define W8_V_CLUSTER (1 << 17)
#define W8_V_BM64 (1 << 18)
#define W8_V_PFIX (1 << 19)
#define W8_V_FUSED (1 << 24)
#define W8_V_PAIR (1 << 25)
#define W8_V_DECODE (1 << 26)
#define W8_V_L2_SHIFT 27
#define W8_V_KPS_SHIFT 20
#define W8_V_CPS_SHIFT 22
#define W8_VARIANT(swap, log2_split, tile, stream)                                            \
    (W8_V_EXPLICIT | ((swap) ? W8_V_SWAP_AB : 0) | ((stream) ? W8_V_STREAM : 0) |            \
     (((log2_split) & 0xF) << W8_V_SPLIT_SHIFT) | (((tile) & 0xF) << W8_V_TILE_SHIFT))

/* ---- entry points ---------------------------------------------------------------- */

/* Dynamic per-token (group == 0) or per-token-group (group == 128) quantization.
 * [FP8] "Kernels Helion implementados": dynamic_per_token_scaled_fp8_quant and
 * per_token_group_fp8_quant; the int8 form is the W8A8 INT8 activation side of [LIN]
 * "Unified GEMM Architecture".
 *   qfmt   W8_Q_FP8 or W8_Q_INT8 (group > 0 and ue8m0 need W8_Q_FP8)
 *   x      bf16 [M, K], row stride ldx >= K; 16-byte aligned, ldx % 8 == 0, K % 8 == 0
 *   q      codes [M, K], row stride K (bytes); 8-byte aligned
 *   scale  fp32 [M] (group == 0) or [M, K/group] (K % group == 0)
 *   ue8m0  nonzero: power-of-two scales (group mode only)
 * Limits: K <= 32768 for group == 0.  Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED, CUDA.
 * Also the offline per-output-channel weight quantizer: pass W[N, K] as x (M = N). */
W8_API int w8_quant_per_token(int qfmt, const void* x, int M, int K, int ldx, void* q, float* scale, int group,
                       int ue8m0, w8_stream_t stream);

/* Block-FP8 weight quantization (offline weight preparation for W8_FMT_BLOCK_FP8*):
 * one scale per 128x128 block of W, s = amax(block)/448 (or its UE8M0 power of two),
 * codes e4m3(w / s).  [FP8] "Kernels Helion implementados" (scaled_mm_blockwise
 * consumes weights in this form).
 *   w      bf16 [N, K] contiguous, 16-byte aligned, K % 8 == 0
 *   q      e4m3 [N, K]; scale fp32 [ceil(N/128), ceil(K/128)] */
W8_API int w8_quant_weight_block(const void* w, int N, int K, void* q, float* scale, int ue8m0, w8_stream_t stream);

/* Fused rms_norm + dynamic per-token fp8 quant, one launch ([FP8] "Patron de fusion
 * del forward pass": rms_norm + fp8_quant; "Kernels Helion implementados":
 * rms_norm_dynamic_per_token_quant).  Per row:
 *   ss = sum x^2, the exact sum rounded once to fp32 (nearest, ties to even; any
 *   summation order gives it); r = 1/sqrt(ss/H + eps) (fp32,
 *   correctly rounded steps); y = (x * r) * gamma in fp32 (never rounded to bf16);
 *   then the per-token fp8 quantization of y.
 *   x bf16 [M, H] (row stride ldx), gamma bf16 [H]; q e4m3 [M, H]; scale fp32 [M].
 * Same alignment rules and limits as w8_quant_per_token (H in place of K). */
W8_API int w8_rmsnorm_quant(const void* x, const void* gamma, float eps, int M, int H, int ldx, void* q, float* scale,
                     w8_stream_t stream);

/* Fused silu_and_mul + dynamic per-token fp8 quant, one launch ([FP8] "Kernels Helion
 * implementados": silu_and_mul_dynamic_per_token_quant).  Row m of gate_up [M, 2I]
 * (row stride ld) holds the gate in columns [0, I) and the up projection in [I, 2I);
 * h = (g / (1 + exp(-g))) * u in fp32 with the library's own correctly specified exp
 * (Cody-Waite reduction, degree-7 polynomial), then per-token fp8 quant of h.
 *   q e4m3 [M, I]; scale fp32 [M].  I % 8 == 0, ld % 8 == 0, 16-byte aligned. */
W8_API int w8_silu_mul_quant(const void* gate_up, int M, int I, int ld, void* q, float* scale, w8_stream_t stream);

/* Per-block fused producers for Block-FP8 ([FP8] "Kernels Helion implementados":
 * rms_norm_per_block_quant, silu_and_mul_per_block_quant): the same fp32 rms_norm /
 * silu_and_mul as above, then fp8 quantization with one scale per 1 x `group` block of
 * each row (group must be 128; H or I a multiple of it), fp32 or UE8M0 (`ue8m0`) scales.
 *   q e4m3 [M, H] or [M, I]; scale fp32 [M, H/128] or [M, I/128] (row-major).
 * Same alignment rules and errors as the per-token producers. */
W8_API int w8_rmsnorm_quant_group(const void* x, const void* gamma, float eps, int M, int H, int ldx, int group,
                                  int ue8m0, void* q, float* scale, w8_stream_t stream);
W8_API int w8_silu_mul_quant_group(const void* gate_up, int M, int I, int ld, int group, int ue8m0, void* q,
                                   float* scale, w8_stream_t stream);

/* Scaled 8-bit GEMM, out = A . W^T with the format's scales, as ONE kernel family whose
 * Standard, Split-K and Swap-AB forms are chosen by `variant` ([LIN] "Unified GEMM
 * Architecture"; [IT] paragraphs 2-3; [FP8] "Kernels Helion implementados":
 * scaled_mm, scaled_mm_blockwise):
 *   FP8_DYN : out[m,n] = bf16( (sum_k a*w) * sA[m] * sW[n] ), fp32 accumulation
 *   INT8    : out[m,n] = bf16( float(sum_k a*w as int32) * sA[m] * sW[n] )
 *   BLOCK   : out[m,n] = bf16( sum_kb sA[m,kb] * sW[n/128,kb] * (sum_{k in kb} a*w) )
 *   A_q      codes [M, K], row-major, 16-byte aligned; K % 16 == 0 (K % 128 for BLOCK)
 *   A_scale  fp32 [M] or [M, K/128] (BLOCK)
 *   W_q      codes [N, K], row-major, 16-byte aligned
 *   W_scale  fp32 [N] or [ceil(N/128), K/128] (BLOCK)
 *   out      bf16 [M, N], row-major
 *   workspace/ws_bytes  scratch for split partials and tile counters, sized by
 *            w8_gemm_workspace_size for the same (fmt, M, N, K, variant), 256-byte
 *            aligned.  Its first 256 KiB hold per-tile counters (the same place for
 *            every shape; at most 65536 output tiles per split call) and must be
 *            zero-filled once before the first use; every successful call leaves them
 *            zero again, so one workspace serves calls of any shape in sequence.  May
 *            be NULL when the size is 0.  Calls that share a workspace must not run
 *            concurrently on the device (successive launches on one stream are fine,
 *            also with W8_V_PDL).  After W8_ERR_DEVICE_TIMEOUT, re-zero it.
 * Accuracy: max|out - ref| <= 2^-7 max|ref| + 1e-3 against the fp64 definition.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, WORKSPACE, NO_DEVICE, CUDA. */
W8_API int w8_gemm(int fmt, const void* A_q, const float* A_scale, const void* W_q, const float* W_scale, void* out,
            int M, int N, int K, int variant, void* workspace, size_t ws_bytes, w8_stream_t stream);

/* Bytes of workspace w8_gemm needs for this call (0 if none); (size_t)-1 if the
 * arguments are invalid.  AUTO is resolved exactly as w8_gemm resolves it. */
W8_API size_t w8_gemm_workspace_size(int fmt, int M, int N, int K, int variant);

/* The explicit variant word AUTO resolves to for this shape (table, else built-in
 * rule), or an explicit `variant` validated and returned unchanged; negative
 * W8_ERR_* if illegal for the shape. */
W8_API int w8_gemm_resolve_variant(int fmt, int M, int N, int K, int variant);

/* INT8 GEMM that writes the raw int32 accumulators acc[M, N] = sum_k a*w (no scales,
 * no bf16), through the same kernels and variants as w8_gemm.  For bit-exact checks
 * of the integer path. */
W8_API int w8_gemm_i32_debug(const void* A_q, const void* W_q, int32_t* acc, int M, int N, int K, int variant,
                      void* workspace, size_t ws_bytes, w8_stream_t stream);

/* Grouped (mixture-of-experts) scaled GEMM.  (The pages name mixture-of-experts models
 * as the next target of the unified linear backend -- "Helion nel backend vLLM: un
 * solo GEMM, tuning per forma e guadagni fino al 10%", last paragraph -- without a
 * formula; this is the plain reading: the experts' GEMMs over tokens already routed.)
 *   A_q [T, K] 8-bit codes, A_scale [T] fp32: the tokens (or token copies, one per
 *       chosen expert) sorted by expert; rows [off[e], off[e+1]) belong to expert e;
 *   expert_offsets int32 [E + 1] in device memory, rising from off[0] >= 0 to off[E]
 *       <= T (read by the kernel after any programmatic-dependent-launch wait, so the
 *       routing kernel ahead may write them); offsets that do not rise within [0, T]
 *       compute nothing and record W8_ERR_INVALID_ARG in the device status word;
 *   W_q [E, N, K] codes, W_scale [E, N] fp32 per expert and output channel;
 *   out [T, N] bf16: row t = bf16(sum_k A[t,k] W_e[n,k] * A_scale[t] * W_scale[e,n]) for
 *       the expert e owning row t (FP8-dynamic or W8A8-INT8, as w8_gemm); rows no expert
 *       owns are not written.
 * The kernel is the Swap-AB GEMM with the balanced partition: every CTA counts the
 * experts' tiles from the offsets and deals out the units of the experts that have
 * tokens, so empty experts cost nothing.  max_tokens_per_expert (<= T) bounds the tokens
 * of one expert; it picks the token tile (AUTO: 16 / 32 / 64, and past 64 tokens the
 * 64-token tile with two CTAs per SM) and sizes the workspace
 * (w8_grouped_gemm_workspace_size; same rules as w8_gemm's).  An explicit variant must
 * be Swap-AB with W8_V_STREAM. */
W8_API int w8_grouped_gemm(int fmt, const void* A_q, const float* A_scale, const void* W_q, const float* W_scale,
                           void* out, const int* expert_offsets, int E, int T, int N, int K,
                           int max_tokens_per_expert, int variant, void* workspace, size_t ws_bytes,
                           w8_stream_t stream);
W8_API size_t w8_grouped_gemm_workspace_size(int fmt, int E, int T, int N, int K, int max_tokens_per_expert,
                                             int variant);

/* Query/key rms_norm + rotary embedding on the merged attention projection ("PyTorch
 * integra Helion en vLLM para acelerar inferencia FP8", section "Kernels Helion
 * implementados": fused_qk_norm_rope; named there without a formula).  Reading:
 *   qkv, out  bf16 [T, (Hq + 2*Hkv) * D] row-major: Hq query heads, Hkv key heads, Hkv
 *             value heads, D contiguous values each; out may equal qkv (in place);
 *   for each token t and query (key) head: y = rms_norm(head) with q_weight (k_weight)
 *             [D] bf16 -- the exact sum of squares rounded once to fp32, r = 1/sqrt(ss/D
 *             + eps), y_k = (x_k * r) * w_k in fp32 -- then each pair (y_i, y_{i+D/2}) is
 *             rotated by the angle of position p = positions[t]: o_i = y_i c_i -
 *             y_{i+D/2} s_i, o_{i+D/2} = y_{i+D/2} c_i + y_i s_i, c_i = cos_sin[p*D + i],
 *             s_i = cos_sin[p*D + D/2 + i] (fp32 table [max_pos, D], the caller's);
 *             rounded to bf16.  Value heads are copied unchanged.
 *   positions int64 [T] in [0, max_pos): a position outside records W8_ERR_INVALID_ARG
 *             in the device status word (w8_device_status) and leaves that token's
 *             query and key heads unwritten.
 * D must be 64, 128 or 256 (W8_ERR_UNSUPPORTED otherwise); qkv, out, the weights and
 * cos_sin 16-byte aligned, positions 8-byte (W8_ERR_ALIGNMENT otherwise). */
W8_API int w8_qk_norm_rope(const void* qkv, void* out, int T, int Hq, int Hkv, int D, const void* q_weight,
                           const void* k_weight, const float* cos_sin, int max_pos, const int64_t* positions,
                           float eps, w8_stream_t stream);

/* Quantize-and-multiply in one call: out = w8_gemm(fmt, quant(x), W) for a bf16
 * activation x [M, K] (row stride ldx elements), with quant the per-token quantizer of
 * w8_quant_per_token for FP8-dynamic (e4m3) and W8A8-INT8 (int8), or its 1 x 128 group
 * form for Block-FP8 (fp32 or UE8M0 scales).  The result is bit-identical to the two
 * calls with the same variant.  ("PyTorch integra Helion en vLLM para acelerar
 * inferencia FP8", section "Patron de fusion del forward pass": the quantizer fused
 * into its neighbour; here the neighbour is the GEMM itself.)
 *   When the resolved variant is Swap-AB with every token in one narrow tile (M <= BN
 *   <= 64), or the decode form (W8_V_DECODE, FP8-dynamic / INT8), ONE kernel can do both:
 *   each CTA reads x, computes the row (or group) maxima -- over its own K range,
 *   exchanged between the ranks of a cluster split, else over the whole row -- and
 *   writes the codes of the K blocks it multiplies straight into shared memory, where
 *   the tensor core reads them (the decode form: in a code region ahead of weight-only
 *   stages, written by the epilogue warps while the weights stream); the quotient x / s
 *   is correctly rounded without a division per element (same codes as the quantizer
 *   kernels).
 *   Otherwise the quantizer kernel runs first into the workspace, then the GEMM (with
 *   programmatic dependent launch when the variant asks for it).  The one-kernel form is
 *   taken only when requested: an explicit variant carrying W8_V_FUSED (W8_ERR_UNSUPPORTED
 *   if it has no fused form), or AUTO when the table's entry carries W8_V_FUSED.  On B200
 *   the two-kernel chain measured faster for every decode shape: the in-kernel
 *   quantization lengthens each CTA's path to its first MMA by more than the quantizer
 *   kernel and its launch cost.
 * x: 16-byte aligned, ldx >= K and a multiple of 8; K as for w8_gemm.  workspace /
 * ws_bytes: at least w8_linear_workspace_size (same rules as w8_gemm's workspace; the
 * two-kernel path keeps the codes and scales there, past the 256 KiB counter area).
 * Errors: as w8_gemm. */
W8_API int w8_linear(int fmt, const void* x, int ldx, const void* W_q, const float* W_scale, void* out, int M, int N,
                     int K, int variant, void* workspace, size_t ws_bytes, w8_stream_t stream);
W8_API size_t w8_linear_workspace_size(int fmt, int M, int N, int K, int variant);
/* The explicit variant w8_linear runs for this shape, with W8_V_FUSED set when it takes
 * the one-kernel form; negative W8_ERR_* if none is legal.  Usable without a device. */
W8_API int w8_linear_resolve(int fmt, int M, int N, int K, int variant);

/* The one-kernel form of w8_linear (W8_V_FUSED implied) that also writes the codes it computed for the K blocks of
 * weight tile 0 (all of K) to q_out [M, K] (16-byte aligned) and the scales to s_out
 * ([M], or [M, K/128] for Block-FP8).  For checking the fused quantization bit for bit;
 * W8_ERR_UNSUPPORTED when the variant has no fused form. */
W8_API int w8_linear_debug(int fmt, const void* x, int ldx, const void* W_q, const float* W_scale, void* out, int M,
                           int N, int K, int variant, void* workspace, size_t ws_bytes, void* q_out, float* s_out,
                           w8_stream_t stream);

/* w8_gemm for callers that cannot allocate device memory.  (An addition of this
 * library: the pages describe no counterpart.)  Some callers cannot provide the
 * Split-K workspace because they may not call cudaMalloc -- code running inside a
 * runtime whose allocator it does not own, or a service whose device memory is fixed
 * at start-up.  This entry point takes the same arguments as w8_gemm minus the
 * workspace and uses instead a scratch array that is part of the library's device
 * code: 8 MiB per GPU, held until the process exits.  A variant whose workspace would
 * exceed that (see w8_gemm_workspace_size) returns W8_ERR_WORKSPACE.  It calls no
 * allocator.  The first call on each device looks up the array's device address; with
 * lazy module loading (CUDA_MODULE_LOADING=LAZY, the default of recent CUDA releases)
 * that lookup is also when the driver places the array -- and the kernels' code -- on
 * the device.  So make one call (any shape or variant) before a memory budget is fixed
 * and before any stream capture.  Each call clears the ticket counters it uses with
 * cudaMemsetAsync on `stream`.  All calls on a device share the array, so calls that
 * overlap on the GPU (e.g. on two streams at once) race; successive calls on one
 * stream are fine.  Errors: as w8_gemm. */
W8_API int w8_gemm_noalloc(int fmt, const void* A_q, const float* A_scale, const void* W_q, const float* W_scale,
                           void* out, int M, int N, int K, int variant, w8_stream_t stream);

/* Failure-path check of the bounded device waits: runs the decode-form GEMM `variant`
 * resolves to (W8_ERR_UNSUPPORTED for other forms) with its producer issuing no loads,
 * so that the tensor core never gets operands, and with every wait bounded by wait_us
 * microseconds (1 .. 1e6) instead of the normal second.  Nothing is ever in flight: the
 * MMA warp's wait for the first stage runs out, the kernel records W8_ERR_DEVICE_TIMEOUT
 * in the device status word (w8_device_status), releases its tensor memory and returns
 * without writing `out`.  The arguments are w8_gemm's (no workspace: the decode form
 * needs none).  Returns the launch status; the timeout shows in w8_device_status once
 * the work has completed.  For testing that a wait which cannot end leaves the GPU and
 * the context usable. */
W8_API int w8_gemm_timeout_debug(int fmt, const void* A_q, const float* A_scale, const void* W_q, const float* W_scale,
                                 void* out, int M, int N, int K, int variant, int wait_us, w8_stream_t stream);

/* Self-check of the quantizers' division-free quotient (every code of w8_quant_per_token,
 * w8_rmsnorm_quant, w8_silu_mul_quant and the fused form of w8_linear is formed from
 * x / s computed with a row reciprocal and Markstein's correction) against the IEEE
 * quotient x / s that defines the codes.  Scale rule: mode % 3 = 0: amax / 448 with e4m3
 * codes, 1: amax / 127 with int8 codes, 2: UE8M0 scales with e4m3 codes.  Modes 0..2
 * enumerate every bf16 amax (smallest subnormal to +inf) and every bf16 x with |x| <= amax,
 * both signs (about 1.1e9 pairs each); modes 3..5 take 2^30 fp32 pairs from a
 * counter-based hash (random finite amax; x random with |x| <= amax, or within 3 ulps of a
 * code's rounding midpoint times s).  A pair fails when the two codes differ, or when the
 * IEEE quotient is at least 2^-10 in magnitude (where a code can depend on it) and the
 * two quotients differ in any bit.  Adds the number
 * of failing pairs to *mismatches; first_bad[0..1] receive (amax bits | 0x80000000, x bits)
 * of one failing pair if first_bad[0] is 0 (bf16 modes: the bf16 patterns in the high
 * halves).  Both are device memory owned by the caller (zero them first); asynchronous on
 * `stream`.  Errors: INVALID_ARG (mode outside 0..5, null pointers), NO_DEVICE, CUDA. */
W8_API int w8_selfcheck_quotient(int mode, unsigned long long* mismatches, unsigned int* first_bad,
                                 w8_stream_t stream);

/* CTAs of the kernel `variant` (AUTO resolved) selects for this shape that can be resident
 * on one SM together, from its registers, shared memory and threads (the CUDA occupancy
 * calculator).  2 or more means a CTA of the next GEMM on the stream can start, and
 * prefetch its weights, beside one of this GEMM while this one finishes.  Returns the
 * count (>= 0) or a negative W8_ERR_*; needs a device. */
W8_API int w8_gemm_occupancy(int fmt, int M, int N, int K, int variant);

/* Per-shape variant table (the output of the offline sweep).  Text, one entry per line:
 *   <fmt> <N> <K> <m_max> <variant as 0x hex>
 * '#' starts a comment.  AUTO picks the entry with the same (fmt, N, K) and the
 * smallest m_max >= M.  Loading replaces the previous table.  Returns the number of
 * entries, or W8_ERR_IO / W8_ERR_INVALID_ARG. */
W8_API int w8_load_table(const char* path);
W8_API void w8_clear_table(void);

/* Device-side error word (set by a kernel whose bounded wait gave up): returns 0 or a
 * W8_ERR_* code for the current device; clears it when `clear` is nonzero.  Reads
 * device memory synchronously: call after the work in question has completed. */
W8_API int w8_device_status(int clear);

W8_API const char* w8_status_string(int status);
W8_API int w8_version(void);

#ifdef __cplusplus
}
#endif
#endif /* W8_H */
