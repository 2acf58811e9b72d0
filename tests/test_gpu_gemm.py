"""GPU parity of the scaled GEMM against the CPU oracle, every format in every variant
(Standard, Split-K, balanced split, Swap-AB; each tile width), at sizes that span
several tiles with ragged edges: bf16 outputs within max|err| <= 2^-7 max|ref| + 1e-3,
INT8 int32 accumulators bit-exact."""
import numpy as np
import pytest
import torch

from bit_quantized_gemm_token_b200 import synth, w8
from gpu_helpers import assert_bf16_close, dev_codes, dev_f32, poison_bf16, quantize_operands

pytestmark = pytest.mark.gpu

SHAPES = [(1, 256, 256), (5, 384, 1024), (16, 300, 640), (17, 1000, 1040), (32, 2048, 1024),
          (33, 256, 512), (64, 1024, 2048), (100, 520, 768), (130, 1024, 2048)]

VARIANTS = {
    "auto": w8.W8_VARIANT_AUTO,
    "swap16": w8.variant(True, 1, 16),
    "swap32_split2": w8.variant(True, 2, 32),
    "swap16_stream": w8.variant(True, 1, 16, stream=True),
    "swap64_split4": w8.variant(True, 4, 64),
    "std128": w8.variant(False, 1, 128),
    "std64_split4": w8.variant(False, 4, 64),
    "std256_stream": w8.variant(False, 1, 256, stream=True),
    "std32_split8": w8.variant(False, 8, 32),
    "swap16_pdl": w8.variant(True, 1, 16, stream=True, pdl=True),
    "swap16_cluster4": w8.variant(True, 4, 16, cluster=True),
    "swap32_cluster2_kps1": w8.variant(True, 2, 32, cluster=True, kps=1),
    "swap16_cluster8_pdl": w8.variant(True, 8, 16, cluster=True, kps=1, pdl=True),
    "std128_cluster2": w8.variant(False, 2, 128, cluster=True),
    "bm64_256_stream": w8.variant(False, 1, 256, stream=True, bm64=True),
    "bm64_128_split2_kps2": w8.variant(False, 2, 128, bm64=True, kps=2, stages=2),
    "bm64_256_cluster2": w8.variant(False, 2, 256, cluster=True, bm64=True, stages=3),
    "bm64_256_split4_pdl": w8.variant(False, 4, 256, bm64=True, stages=2, pdl=True),
    "bm64_256_cluster4": w8.variant(False, 4, 256, cluster=True, bm64=True, stages=3),
    "bm64_128_stream2": w8.variant(False, 1, 128, stream=True, bm64=True, cps=2, stages=2),
    "bm64_256_stream_pfix": w8.variant(False, 1, 256, stream=True, bm64=True, pfix=True),
    "bm64_256_stream_pfix_pdl": w8.variant(False, 1, 256, stream=True, bm64=True, pfix=True, pdl=True, kps=1, stages=5),
    "bm64_128_split4_pfix_kps2": w8.variant(False, 4, 128, bm64=True, pfix=True, kps=2, stages=3),
    "bm64_256_split2_pfix": w8.variant(False, 2, 256, bm64=True, pfix=True, kps=1),
    "pair256": w8.variant(False, 1, 256, pair=True),
    "pair256_st3_pdl": w8.variant(False, 1, 256, pair=True, stages=3, pdl=True),
}

BLOCK_OK = {"auto", "swap16", "swap32_split2", "swap16_stream", "swap64_split4", "std64_split4", "std32_split8",
            "swap16_pdl", "swap16_cluster4", "swap32_cluster2_kps1", "swap16_cluster8_pdl"}

_cache = {}


def operands(orc, fmt, M, N, K, ue8m0=False):
    key = (fmt, M, N, K, ue8m0)
    if key not in _cache:
        x = synth.activations(M, K, seed=10_000 + M * 31 + K)
        w = synth.weights(N, K, seed=20_000 + N * 7 + K)
        Aq, sA, Wq, sW = quantize_operands(orc, fmt if fmt < 2 else 2, x, w, ue8m0)
        ofmt = 2 if fmt >= 2 else fmt
        out, ref, acc = orc.gemm(ofmt, Aq, sA, Wq, sW)
        _cache[key] = (Aq, sA, Wq, sW, ref, acc)
    return _cache[key]


def run(fmt, Aq, sA, Wq, sW, v, M, N):
    cf = 1 if fmt == 1 else 0
    out = poison_bf16((M, N))
    w8.w8_gemm(fmt, dev_codes(Aq, cf), dev_f32(sA), dev_codes(Wq, cf), dev_f32(sW), out=out, variant=v)
    torch.cuda.synchronize()
    return out


def legal(fmt, M, N, K, v):
    try:
        w8.w8_gemm_resolve_variant(fmt, M, N, K, v)
        return True
    except w8.W8Error:
        return False


@pytest.mark.parametrize("vname", list(VARIANTS))
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_fp8_dynamic(orc, M, N, K, vname):
    v = VARIANTS[vname]
    if not legal(0, M, N, K, v):
        pytest.skip("variant illegal for shape")
    Aq, sA, Wq, sW, ref, _ = operands(orc, 0, M, N, K)
    assert_bf16_close(run(0, Aq, sA, Wq, sW, v, M, N), ref, "fp8 %s %s" % (vname, (M, N, K)))


@pytest.mark.parametrize("vname", list(VARIANTS))
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_int8_accumulators_exact(orc, M, N, K, vname):
    v = VARIANTS[vname]
    if not legal(1, M, N, K, v):
        pytest.skip("variant illegal for shape")
    Aq, sA, Wq, sW, ref, acc = operands(orc, 1, M, N, K)
    got = w8.w8_gemm_i32_debug(dev_codes(Aq, 1), dev_codes(Wq, 1), variant=v)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy().astype(np.int64), acc)
    assert_bf16_close(run(1, Aq, sA, Wq, sW, v, M, N), ref, "int8 %s %s" % (vname, (M, N, K)))


BLOCK_SHAPES = [(1, 256, 256), (5, 384, 1024), (16, 300, 640), (32, 1024, 1152), (33, 256, 512), (100, 520, 768)]


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("vname", sorted(BLOCK_OK))
@pytest.mark.parametrize("M,N,K", BLOCK_SHAPES)
def test_block_fp8(orc, M, N, K, vname, ue8m0):
    v = VARIANTS[vname]
    fmt = w8.W8_FMT_BLOCK_FP8_UE8M0 if ue8m0 else w8.W8_FMT_BLOCK_FP8
    if not legal(fmt, M, N, K, v):
        pytest.skip("variant illegal for shape")
    Aq, sA, Wq, sW, ref, _ = operands(orc, fmt, M, N, K, ue8m0)
    assert_bf16_close(run(fmt, Aq, sA, Wq, sW, v, M, N), ref, "block %s %s" % (vname, (M, N, K)))


def test_split_k_up_to_256(orc):
    """Power-of-two splits up to 256 (K = 32768 has 256 K blocks)."""
    M, N, K = 8, 256, 32768
    Aq, sA, Wq, sW, ref, acc = operands(orc, 1, M, N, K)
    for S in (1, 2, 16, 64, 256):
        for swap, bn in ((True, 16), (False, 128)):
            v = w8.variant(swap, S, bn)
            got = w8.w8_gemm_i32_debug(dev_codes(Aq, 1), dev_codes(Wq, 1), variant=v)
            torch.cuda.synchronize()
            assert np.array_equal(got.cpu().numpy().astype(np.int64), acc), (S, swap)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("M,N,K", [(1000, 5000, 384), (300, 40000, 256), (4096, 2048, 272), (257, 257, 128)])
def test_pair_tiles(orc, fmt, M, N, K):
    """256 x 256 tiles on CTA pairs at sizes with more tiles than pairs, ragged token and
    weight tiles and a ragged K block: the oracle's outputs within the GEMM bound and,
    for INT8, its int32 accumulators exactly."""
    Aq, sA, Wq, sW, ref, acc = operands(orc, fmt, M, N, K)
    for v in (w8.variant(False, 1, 256, pair=True), w8.variant(False, 1, 256, pair=True, pdl=True, stages=4)):
        assert_bf16_close(run(fmt, Aq, sA, Wq, sW, v, M, N), ref, "pair %s" % ((M, N, K),))
        if fmt == 1:
            a32 = w8.w8_gemm_i32_debug(dev_codes(Aq, 1), dev_codes(Wq, 1), variant=v)
            torch.cuda.synchronize()
            assert np.array_equal(a32.cpu().numpy().astype(np.int64), acc)
    assert w8.w8_device_status(clear=True) == 0


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("M,N,K", [(300, 600, 2048), (256, 512, 1040), (64, 300, 4096), (513, 256, 1024)])
def test_pair_split_k(orc, fmt, M, N, K):
    """CTA-pair tiles with a K split (one (tile, K chunk) unit per pair, the last
    contributor adding the chunks in order): ragged token, weight and K tiles, split up
    to one K block per chunk; the oracle's outputs within the GEMM bound, INT8 int32
    accumulators exactly, and the same bytes on a second call with the same workspace."""
    Aq, sA, Wq, sW, ref, acc = operands(orc, fmt, M, N, K)
    A, SA, W, SW = dev_codes(Aq, fmt), dev_f32(sA), dev_codes(Wq, fmt), dev_f32(sW)
    tiles = -(-M // 256) * -(-N // 256)
    kbs = -(-K // 128)
    ws = w8.Workspace()
    ran = 0
    for S in (2, 4, 8):
        if tiles * S > 74 or S > kbs:
            with pytest.raises(w8.W8Error):
                w8.w8_gemm_resolve_variant(fmt, M, N, K, w8.variant(False, S, 256, pair=True))
            continue
        for v in (w8.variant(False, S, 256, pair=True), w8.variant(False, S, 256, pair=True, pdl=True, stages=3)):
            o1 = w8.w8_gemm(fmt, A, SA, W, SW, variant=v, workspace=ws).clone()
            o2 = w8.w8_gemm(fmt, A, SA, W, SW, variant=v, workspace=ws).clone()
            torch.cuda.synchronize()
            assert_bf16_close(o1, ref, "pair split %d %s" % (S, (M, N, K)))
            assert torch.equal(o1, o2)
            if fmt == 1:
                a32 = w8.w8_gemm_i32_debug(A, W, variant=v, workspace=ws)
                torch.cuda.synchronize()
                assert np.array_equal(a32.cpu().numpy().astype(np.int64), acc)
            ran += 1
    assert ran > 0
    assert int(ws.buf[:256 * 1024].sum()) == 0      # counter area back to zero
    assert w8.w8_device_status(clear=True) == 0


def test_repeated_calls_reuse_workspace(orc):
    """Counters are left at zero: the same workspace serves back-to-back split calls,
    and the results are bit-identical run to run (fixed reduction order)."""
    M, N, K = 16, 2048, 4096
    Aq, sA, Wq, sW, ref, _ = operands(orc, 0, M, N, K)
    ws = w8.Workspace()
    A, SA, W, SW = dev_codes(Aq, 0), dev_f32(sA), dev_codes(Wq, 0), dev_f32(sW)
    outs = []
    for v in [w8.variant(True, 8, 16), w8.variant(True, 1, 16, stream=True),
              w8.variant(False, 1, 256, stream=True, bm64=True, pfix=True)] * 3:
        outs.append(w8.w8_gemm(0, A, SA, W, SW, variant=v, workspace=ws).clone())
    torch.cuda.synchronize()
    for o in outs:
        assert_bf16_close(o, ref, "repeat")
    assert torch.equal(outs[0], outs[3]) and torch.equal(outs[1], outs[4]) and torch.equal(outs[2], outs[5])
    assert int(ws.buf[:256].sum()) == 0      # counter area back to zero
    assert w8.w8_device_status(clear=True) == 0


def test_workspace_too_small_is_rejected(orc):
    import ctypes
    M, N, K = 4, 256, 1024
    Aq, sA, Wq, sW, ref, _ = operands(orc, 0, M, N, K)
    v = w8.variant(True, 4, 16)
    need = w8.w8_gemm_workspace_size(0, M, N, K, v)
    assert need > 256
    small = torch.zeros(need - 256, dtype=torch.uint8, device="cuda")
    A, SA, W, SW = dev_codes(Aq, 0), dev_f32(sA), dev_codes(Wq, 0), dev_f32(sW)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = w8.lib().w8_gemm(0, P(A), P(SA), P(W), P(SW), P(out), M, N, K, v, P(small), small.numel(), s)
    assert rc == w8.W8_ERR_WORKSPACE
    rc = w8.lib().w8_gemm(0, P(A), P(SA), P(W), P(SW), P(out), M, N, K, v, None, 0, s)
    assert rc == w8.W8_ERR_WORKSPACE


def test_graph_capture_small_m(orc):
    """Decode-sized launches replayed from a CUDA graph give the same bytes."""
    M, N, K = 4, 1024, 2048
    Aq, sA, Wq, sW, ref, _ = operands(orc, 0, M, N, K)
    A, SA, W, SW = dev_codes(Aq, 0), dev_f32(sA), dev_codes(Wq, 0), dev_f32(sW)
    ws = w8.Workspace(nbytes=w8.w8_gemm_workspace_size(0, M, N, K, 0))
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        w8.w8_gemm(0, A, SA, W, SW, out=out, workspace=ws)
    torch.cuda.synchronize()
    eager = out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        w8.w8_gemm(0, A, SA, W, SW, out=out, workspace=ws, variant=w8.W8_V_PDL)
    out.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
    assert_bf16_close(out, ref, "graph")


def test_workspace_shared_across_shapes(orc):
    """One workspace for calls of different shapes in sequence: the partial sums of a
    call with few tiles must not be read as ticket counters by a call with many."""
    ws = w8.Workspace()
    for (M, N, K, v) in [(16, 256, 4096, w8.variant(True, 32, 16)), (1, 8192, 1024, w8.variant(True, 1, 16, stream=True)),
                         (3, 512, 2048, w8.variant(True, 16, 16)), (1, 8192, 1024, w8.variant(True, 1, 16, stream=True))]:
        Aq, sA, Wq, sW, ref, _ = operands(orc, 0, M, N, K)
        out = poison_bf16((M, N))
        w8.w8_gemm(0, dev_codes(Aq, 0), dev_f32(sA), dev_codes(Wq, 0), dev_f32(sW), out=out, variant=v, workspace=ws)
        torch.cuda.synchronize()
        assert_bf16_close(out, ref, "shared workspace %s" % ((M, N, K),))
    assert int(ws.buf[:65536 * 4].sum()) == 0


def test_occupancy_query():
    """The occupancy query answers for every family; a 6-warp CTA above 128 registers
    per thread holds an SM alone (the register file is split per scheduler)."""
    for fmt, M, N, K, v in [(0, 1, 4096, 4096, w8.variant(True, 4, 16, cluster=True)),
                            (1, 8, 4096, 4096, w8.variant(True, 1, 16, stream=True)),
                            (2, 4, 6144, 4096, w8.variant(True, 1, 32, stream=True)),
                            (0, 8, 4096, 4096, w8.variant(False, 1, 256, stream=True, bm64=True))]:
        n = w8.w8_gemm_occupancy(fmt, M, N, K, v)
        assert n >= 1
    with pytest.raises(w8.W8Error):
        w8.w8_gemm_occupancy(0, 8, 256, 256, w8.variant(True, split=4, bn=16))
