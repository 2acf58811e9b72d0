"""GPU parity of the decode form of the scaled GEMM (W8_V_DECODE: tokens in the 64-row
MMA operand, 64..256 weight rows per tile, K split over a thread-block cluster and
reduced in distributed shared memory) against the CPU oracle: FP8-dynamic outputs
within max|err| <= 2^-7 max|ref| + 1e-3, W8A8-INT8 int32 accumulators bit-exact, at
sizes with ragged token boxes, ragged weight tiles, ragged K blocks and chunk counts
that do not divide the K blocks."""
import numpy as np
import pytest
import torch

from bit_quantized_gemm_token_b200 import synth, w8
from gpu_helpers import assert_bf16_close, dev_codes, dev_f32, poison_bf16, quantize_operands

pytestmark = pytest.mark.gpu

SHAPES = [(1, 256, 256), (5, 300, 640), (16, 1000, 1040), (17, 2048, 4096), (32, 520, 1536), (33, 256, 512),
          (64, 1024, 2048), (8, 4096, 4096)]

DECODE = {
    "bn256_c1": dict(bn=256, c=1),
    "bn256_c8": dict(bn=256, c=8),
    "bn128_c4_st2": dict(bn=128, c=4, stages=2),
    "bn64_c2_l2_0": dict(bn=64, c=2, l2ahead=0),
    "bn176_c3_pdl": dict(bn=176, c=3, pdl=True),
    "bn240_c6_st4": dict(bn=240, c=6, stages=4),
    "bn256_c5_pdl_l2_8": dict(bn=256, c=5, pdl=True, l2ahead=8),
    "bn96_c7": dict(bn=96, c=7),
}

_cache = {}


def operands(orc, fmt, M, N, K):
    key = (fmt, M, N, K)
    if key not in _cache:
        x = synth.activations(M, K, seed=30_000 + M * 31 + K)
        w = synth.weights(N, K, seed=40_000 + N * 7 + K)
        Aq, sA, Wq, sW = quantize_operands(orc, fmt, x, w)
        _, ref, acc = orc.gemm(fmt, Aq, sA, Wq, sW)
        _cache[key] = (Aq, sA, Wq, sW, ref, acc)
    return _cache[key]


def legal(fmt, M, N, K, v):
    try:
        w8.w8_gemm_resolve_variant(fmt, M, N, K, v)
        return True
    except w8.W8Error:
        return False


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("vname", list(DECODE))
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_decode_form(orc, fmt, M, N, K, vname):
    v = w8.decode_variant(**DECODE[vname])
    if not legal(fmt, M, N, K, v):
        pytest.skip("variant illegal for shape")
    Aq, sA, Wq, sW, ref, acc = operands(orc, fmt, M, N, K)
    A, W = dev_codes(Aq, fmt), dev_codes(Wq, fmt)
    out = poison_bf16((M, N))
    w8.w8_gemm(fmt, A, dev_f32(sA), W, dev_f32(sW), out=out, variant=v)
    torch.cuda.synchronize()
    assert_bf16_close(out, ref, "decode %s fmt %d %s" % (vname, fmt, (M, N, K)))
    if fmt == 1:
        got = w8.w8_gemm_i32_debug(A, W, variant=v)
        torch.cuda.synchronize()
        assert np.array_equal(got.cpu().numpy().astype(np.int64), acc)
    assert w8.w8_device_status(clear=True) == 0


def test_decode_repeatable_and_chained(orc):
    """Back-to-back launches with programmatic dependent launch on one stream (the next
    GEMM's CTAs start beside the current ones) give bit-identical results run to run."""
    M, N, K = 16, 2048, 4096
    Aq, sA, Wq, sW, ref, _ = operands(orc, 0, M, N, K)
    A, SA, W, SW = dev_codes(Aq, 0), dev_f32(sA), dev_codes(Wq, 0), dev_f32(sW)
    outs = [poison_bf16((M, N)) for _ in range(6)]
    vs = [w8.decode_variant(256, 8, pdl=True), w8.decode_variant(128, 2, pdl=True, stages=2),
          w8.decode_variant(256, 1, pdl=True, l2ahead=6)] * 2
    for o, v in zip(outs, vs):
        w8.w8_gemm(0, A, SA, W, SW, out=o, variant=v)
    torch.cuda.synchronize()
    for o in outs:
        assert_bf16_close(o, ref, "chained decode")
    for i in range(3):
        assert torch.equal(outs[i], outs[i + 3])
    assert w8.w8_device_status(clear=True) == 0


def test_decode_rejects_illegal():
    with pytest.raises(w8.W8Error):
        w8.w8_gemm_resolve_variant(0, 65, 1024, 1024, w8.decode_variant(256, 1))    # more than 64 tokens
    with pytest.raises(w8.W8Error):
        w8.w8_gemm_resolve_variant(0, 8, 1024, 256, w8.decode_variant(256, 3))      # 3 chunks of 2 K blocks
    with pytest.raises(w8.W8Error):
        w8.w8_gemm_resolve_variant(2, 8, 1024, 1024, w8.decode_variant(256, 1))     # Block-FP8
