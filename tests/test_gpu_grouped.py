"""GPU parity of the grouped (mixture-of-experts) GEMM with the CPU oracle: decode-like
routings (few experts with tokens, many empty), an expert with more tokens than one
token tile, FP8-dynamic and INT8, every token-tile width, programmatic dependent
launch; rows no expert owns stay untouched; bad offsets compute nothing and are
reported."""
import numpy as np
import pytest
import torch

from bit_quantized_gemm_token_b200 import synth, w8
from gpu_helpers import assert_bf16_close, bits, dev_codes, dev_f32

pytestmark = pytest.mark.gpu


def make(orc, fmt, counts, N, K, seed, extra_rows=0):
    E = len(counts)
    T = int(sum(counts)) + extra_rows
    x = synth.activations(T, K, seed=seed)
    Aq, sA = orc.quant_rows(fmt, bits(x))
    Wq = np.zeros((E, N, K), dtype=np.int8 if fmt == 1 else np.uint8)
    sW = np.zeros((E, N), dtype=np.float32)
    for e in range(E):
        q, s = orc.quant_rows(fmt, bits(synth.weights(N, K, seed=seed + 100 + e)))
        Wq[e], sW[e] = q, s
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return Aq, sA, Wq, sW, off


def run(orc, fmt, counts, N, K, variant=w8.W8_VARIANT_AUTO, seed=1, extra_rows=0, mm=None):
    Aq, sA, Wq, sW, off = make(orc, fmt, counts, N, K, seed, extra_rows)
    T = Aq.shape[0]
    cf = 1 if fmt == 1 else 0
    Wd = dev_codes(Wq.reshape(-1, K), cf).view(len(counts), N, K)
    out = torch.full((T, N), 7.0, dtype=torch.bfloat16, device="cuda")
    w8.w8_grouped_gemm(fmt, dev_codes(Aq, cf), dev_f32(sA), Wd, dev_f32(sW), torch.from_numpy(off).cuda(),
                       max_tokens_per_expert=(mm if mm is not None else max(max(counts), 1)), out=out, variant=variant)
    torch.cuda.synchronize()
    _, ref, _ = orc.grouped_gemm(fmt, Aq, sA, Wq, sW, off)
    owned = int(off[-1])
    if owned:
        assert_bf16_close(out[:owned], ref[:owned], "grouped fmt %d counts %s" % (fmt, counts))
    assert torch.all(out[owned:] == 7.0)
    assert w8.w8_device_status(clear=True) == 0
    return out


ROUTINGS = {
    "decode_top8_of_64": [1 if e in (3, 7, 8, 20, 33, 41, 50, 63) else 0 for e in range(64)],
    "decode_4tok_top2_of_16": [0, 2, 0, 1, 0, 0, 3, 0, 0, 1, 0, 0, 0, 1, 0, 0],
    "uneven_8": [5, 0, 17, 1, 0, 0, 40, 2],
    "one_big_expert": [0, 70, 3],
    "single_expert": [9],
}


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("name", list(ROUTINGS))
@pytest.mark.parametrize("N,K", [(256, 1024), (768, 2048)])
def test_routings(orc, fmt, name, N, K):
    run(orc, fmt, ROUTINGS[name], N, K, seed=10 + len(name) + N // 128)


@pytest.mark.parametrize("variant", [w8.variant(True, 1, 16, stream=True), w8.variant(True, 1, 32, stream=True, pdl=True),
                                     w8.variant(True, 1, 64, stream=True, cps=2), w8.variant(True, 1, 16, stream=True, kps=1)])
def test_variants(orc, variant):
    run(orc, 0, ROUTINGS["uneven_8"], 384, 1024, variant=variant, seed=77)


def test_rows_past_last_offset_untouched(orc):
    run(orc, 0, [2, 0, 3], 256, 512, seed=81, extra_rows=5)


def test_repeatable(orc):
    a = run(orc, 0, ROUTINGS["uneven_8"], 256, 1024, seed=83)
    b = run(orc, 0, ROUTINGS["uneven_8"], 256, 1024, seed=83)
    assert torch.equal(a, b)


def test_bad_offsets_compute_nothing(orc):
    T, N, K, E = 8, 256, 512, 3
    A = torch.zeros((T, K), dtype=torch.float8_e4m3fn, device="cuda")
    W = torch.zeros((E, N, K), dtype=torch.float8_e4m3fn, device="cuda")
    sA = torch.ones(T, device="cuda")
    sW = torch.ones((E, N), device="cuda")
    out = torch.full((T, N), 7.0, dtype=torch.bfloat16, device="cuda")
    off = torch.tensor([0, 5, 3, 8], dtype=torch.int32, device="cuda")   # falls back
    w8.w8_device_status(clear=True)
    w8.w8_grouped_gemm(0, A, sA, W, sW, off, max_tokens_per_expert=8, out=out)
    torch.cuda.synchronize()
    assert w8.w8_device_status(clear=True) == w8.W8_ERR_INVALID_ARG
    assert torch.all(out == 7.0)


PREFILL_ROUTING = [300, 0, 513, 129, 260, 77]


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("variant", [w8.W8_VARIANT_AUTO, w8.variant(True, 1, 128, stream=True),
                                     w8.variant(True, 1, 256, stream=True, pdl=True),
                                     w8.variant(True, 1, 256, stream=True, kps=1)])
def test_prefill_routing(orc, fmt, variant):
    """Hundreds of tokens per expert (several 128- or 256-token tiles per expert, ragged
    last tiles, an empty expert, an expert whose token box must start before its first
    row near the end of A): the oracle's outputs, untouched rows past the last offset."""
    run(orc, fmt, PREFILL_ROUTING, 384, 1024, variant=variant, seed=91 + fmt, extra_rows=3)
