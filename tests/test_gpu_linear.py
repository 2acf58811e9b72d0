"""GPU parity of w8_linear, the quantizer fused into the GEMM (the Swap-AB form and the
decode form): the codes and scales the kernel computes itself equal the oracle's bit for
bit, the outputs equal those of the
two-kernel path (quantizer, then GEMM) with the same variant bit for bit, and both meet
the GEMM tolerance against the oracle."""
import numpy as np
import pytest
import torch

from bit_quantized_gemm_token_b200 import synth, w8
from gpu_helpers import assert_bf16_close, bits, dev_codes, dev_f32, u8

pytestmark = pytest.mark.gpu

FUSED = {
    "swap16": w8.variant(True, 1, 16),
    "swap16_stream": w8.variant(True, 1, 16, stream=True),
    "swap16_split4": w8.variant(True, 4, 16),
    "swap16_cluster4": w8.variant(True, 4, 16, cluster=True),
    "swap32_cluster2_kps1": w8.variant(True, 2, 32, cluster=True, kps=1),
    "swap32_stream_pdl": w8.variant(True, 1, 32, stream=True, pdl=True),
    "swap64_split2": w8.variant(True, 2, 64),
    "swap16_cluster8": w8.variant(True, 8, 16, cluster=True, kps=1),
    # the decode form: the epilogue warps quantize the rank's K blocks into a code region
    # while the weights stream; row maxima exchanged between the K-chunk ranks
    "decode_bn256_c1": w8.decode_variant(256, 1),
    "decode_bn128_c4": w8.decode_variant(128, 4),
    "decode_bn176_c3_pdl": w8.decode_variant(176, 3, pdl=True),
    "decode_bn64_c8_st2": w8.decode_variant(64, 8, stages=2),
}

# (M, N, K): several weight tiles, a ragged last K block (1040), a K range wider than a
# stage ring, and the decode sizes
SHAPES = [(1, 256, 1024), (3, 384, 1040), (16, 512, 2048), (29, 256, 4096), (1, 1024, 12288), (64, 256, 512)]


def fused_ok(fmt, M, N, K, v):
    try:
        w8.w8_gemm_resolve_variant(fmt, M, N, K, v)
    except w8.W8Error:
        return False
    try:
        x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
        W = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
        sw = torch.ones(N if fmt < 2 else (N + 127) // 128 * (K // 128), device="cuda")
        w8.w8_linear(fmt, x, W, sw, variant=v | w8.W8_V_FUSED)
        return True
    except w8.W8Error as e:
        if e.code == w8.W8_ERR_UNSUPPORTED:
            return False
        raise


def weights(orc, fmt, N, K, ue8m0=False):
    w = synth.weights(N, K, seed=21_000 + N + K)
    if fmt == 2:
        Wq, sW = orc.quant_weight_block(bits(w), ue8m0=ue8m0)
    else:
        Wq, sW = orc.quant_rows(fmt, bits(w))
    return Wq, sW


def check_codes(orc, fmt, x, q, s, ue8m0=False):
    if fmt == 2:
        oq, os_ = orc.quant_rows(0, bits(x), group=128, ue8m0=ue8m0)
    else:
        oq, os_ = orc.quant_rows(fmt, bits(x))
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(u8(q), np.ascontiguousarray(oq).view(np.uint8))


@pytest.mark.parametrize("vname", list(FUSED))
@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("fmt", [0, 1, 2, 3])
def test_fused_codes_and_outputs(orc, fmt, M, N, K, vname):
    v = FUSED[vname]
    if fmt >= 2 and K % 128 != 0:
        pytest.skip("Block-FP8 needs K % 128 == 0")
    if not fused_ok(fmt, M, N, K, v):
        pytest.skip("no fused form for this variant and shape")
    ue8m0 = fmt == 3
    ofmt = 2 if fmt >= 2 else fmt
    x = synth.activations(M, K, seed=30_000 + M * 13 + K)
    Wq, sW = weights(orc, ofmt, N, K, ue8m0)
    cf = 1 if fmt == 1 else 0
    Wd, sWd = dev_codes(Wq, cf), dev_f32(sW)
    xd = x.cuda()
    out, q, s = w8.w8_linear_debug(fmt, xd, Wd, sWd, variant=v)
    torch.cuda.synchronize()
    check_codes(orc, ofmt, x, q, s, ue8m0)
    # the same variant through the two-kernel path: identical bytes
    two = w8.w8_linear(fmt, xd, Wd, sWd, variant=v)
    fused = w8.w8_linear(fmt, xd, Wd, sWd, variant=v | w8.W8_V_FUSED)
    torch.cuda.synchronize()
    assert torch.equal(fused, out)
    assert torch.equal(fused, two)
    # against the oracle's GEMM on the oracle's codes
    if fmt >= 2:
        Aq, sA = orc.quant_rows(0, bits(x), group=128, ue8m0=ue8m0)
    else:
        Aq, sA = orc.quant_rows(fmt, bits(x))
    _, ref, _ = orc.gemm(ofmt, Aq, sA, Wq, sW)
    assert_bf16_close(fused, ref, "fused %s fmt %d" % (vname, fmt))


def test_fused_special_rows(orc):
    """All-zero rows (s = 1), signed zeros, tiny rows whose scale is subnormal, and a
    strided x: the codes still equal the oracle's."""
    M, N, K = 6, 256, 1024
    big = synth.activations(M, K + 64, seed=31_000)
    big[1] = 0.0
    big[2, :] = -0.0
    big[3] = big[3] * 1e-37          # amax / 448 below the fp32 normal range
    big[4, ::7] = -0.0
    xd = big.cuda()[:, :K]
    x = big[:, :K].contiguous()
    for fmt in (0, 1, 2, 3):
        ofmt = 2 if fmt >= 2 else fmt
        Wq, sW = weights(orc, ofmt, N, K, fmt == 3)
        cf = 1 if fmt == 1 else 0
        v = w8.variant(True, 4, 16, cluster=True)
        out, q, s = w8.w8_linear_debug(fmt, xd, dev_codes(Wq, cf), dev_f32(sW), variant=v)
        torch.cuda.synchronize()
        check_codes(orc, ofmt, x, q, s, fmt == 3)


def test_auto_and_two_kernel_paths(orc):
    """AUTO (no table entry asking for the fused form) runs the quantizer and the GEMM:
    the same bytes as the two calls, for a Swap-AB and a Standard (M = 100) variant."""
    for M in (2, 100):
        N, K = 512, 2048
        x = synth.activations(M, K, seed=32_000 + M)
        Wq, sW = weights(orc, 0, N, K)
        Wd, sWd, xd = dev_codes(Wq, 0), dev_f32(sW), x.cuda()
        got = w8.w8_linear(0, xd, Wd, sWd)
        q, s = w8.w8_quant_per_token(xd, w8.W8_Q_FP8)
        v = w8.w8_gemm_resolve_variant(0, M, N, K)
        ref = w8.w8_gemm(0, q, s, Wd, sWd, variant=v)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), M


def test_explicit_variant_without_fused_form_is_rejected(orc):
    M, N, K = 8, 256, 1024
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((N, K), dtype=torch.float8_e4m3fn, device="cuda")
    sw = torch.ones(N, device="cuda")
    with pytest.raises(w8.W8Error) as e:
        w8.w8_linear(0, x, W, sw, variant=w8.variant(False, 1, 128) | w8.W8_V_FUSED)
    assert e.value.code == w8.W8_ERR_UNSUPPORTED
    w8.w8_linear(0, x, W, sw, variant=w8.variant(False, 1, 128))
    torch.cuda.synchronize()
    assert w8.w8_device_status(clear=True) == 0


def test_two_kernel_path_keeps_counters_zero(orc):
    """The two-kernel path stores the codes in the workspace: never inside the counter
    area that split GEMMs sharing the workspace rely on (a variant without partials
    would otherwise put them at offset 0)."""
    ws = w8.Workspace()
    M, N, K = 64, 256, 2048
    x = synth.activations(M, K, seed=33_000)
    Wq, sW = weights(orc, 0, N, K)
    Wd, sWd, xd = dev_codes(Wq, 0), dev_f32(sW), x.cuda()
    w8.w8_linear(0, xd, Wd, sWd, variant=w8.variant(False, 1, 128), workspace=ws)
    torch.cuda.synchronize()
    assert int(ws.buf[:65536 * 4].view(torch.int32).abs().sum()) == 0
    Aq, sA = orc.quant_rows(0, bits(x))
    _, ref, _ = orc.gemm(0, Aq, sA, Wq, sW)
    out = w8.w8_linear(0, xd, Wd, sWd, variant=w8.variant(True, 2, 64), workspace=ws)
    torch.cuda.synchronize()
    assert_bf16_close(out, ref, "split after unfused")
