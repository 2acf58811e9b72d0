"""Pins of the oracle's scaled GEMM: int8 against numpy's exact int64 matmul, fp8 against
an fp64 matmul of torch-decoded operands, Block-FP8 against a per-block numpy
formulation and against FP8-dynamic when the block scales are uniform, brute force on
tiny shapes, and the Swap-AB and Split-K identities."""
import itertools

import numpy as np
import pytest
import torch

from bit_quantized_gemm_token_b200 import synth


def decode_fp8(q):
    return torch.from_numpy(np.ascontiguousarray(q, dtype=np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def operands(orc, fmt, M, N, K, seed, ue8m0=False):
    x = synth.activations(M, K, seed=seed)
    w = synth.weights(N, K, seed=seed + 1)
    if fmt == 0:
        Aq, sA = orc.quant_rows(0, synth.bf16_bits(x))
        Wq, sW = orc.quant_rows(0, synth.bf16_bits(w))
    elif fmt == 1:
        Aq, sA = orc.quant_rows(1, synth.bf16_bits(x))
        Wq, sW = orc.quant_rows(1, synth.bf16_bits(w))
    else:
        Aq, sA = orc.quant_rows(0, synth.bf16_bits(x), group=128, ue8m0=ue8m0)
        Wq, sW = orc.quant_weight_block(synth.bf16_bits(w), ue8m0=ue8m0)
    return Aq, sA, Wq, sW


@pytest.mark.parametrize("M,N,K", [(1, 256, 1024), (16, 384, 1024), (32, 200, 640), (3, 130, 4096)])
def test_int8_exact_against_numpy(orc, M, N, K):
    Aq, sA, Wq, sW = operands(orc, 1, M, N, K, seed=100 + M)
    out, ref, acc = orc.gemm(1, Aq, sA, Wq, sW)
    want = Aq.astype(np.int64) @ Wq.astype(np.int64).T
    assert np.array_equal(acc, want)
    assert np.all(np.abs(want) < 2 ** 31)
    assert np.allclose(ref, want * sA[:, None].astype(np.float64) * sW[None, :].astype(np.float64), rtol=1e-15, atol=0)


@pytest.mark.parametrize("M,N,K", [(1, 256, 1024), (16, 384, 1024), (5, 130, 4096)])
def test_fp8_against_fp64_matmul(orc, M, N, K):
    Aq, sA, Wq, sW = operands(orc, 0, M, N, K, seed=200 + M)
    out, ref, _ = orc.gemm(0, Aq, sA, Wq, sW)
    want = (decode_fp8(Aq) @ decode_fp8(Wq).T) * sA[:, None].astype(np.float64) * sW[None, :].astype(np.float64)
    assert np.allclose(ref, want, rtol=1e-13, atol=0)
    ok, err, bound = orc.bf16_max_err_ok(out, want)
    assert ok
    # bf16 output is the one-time RNE rounding of the fp64 result
    tb = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.mean(out == tb) > 0.999


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (9, 384, 1024), (32, 128, 256)])
def test_block_against_numpy_blocks(orc, M, N, K, ue8m0):
    Aq, sA, Wq, sW = operands(orc, 2, M, N, K, seed=300 + M, ue8m0=ue8m0)
    out, ref, _ = orc.gemm(2, Aq, sA, Wq, sW)
    a, w = decode_fp8(Aq), decode_fp8(Wq)
    want = np.zeros((M, N))
    for kb in range(K // 128):
        part = a[:, kb * 128:(kb + 1) * 128] @ w[:, kb * 128:(kb + 1) * 128].T
        sw = np.repeat(sW[:, kb].astype(np.float64), 128)[:N]
        want += part * sA[:, kb, None].astype(np.float64) * sw[None, :]
    assert np.allclose(ref, want, rtol=1e-12, atol=0)
    if ue8m0:
        assert np.all(np.frexp(sA)[0] == 0.5) and np.all(np.frexp(sW)[0] == 0.5)


def test_block_with_uniform_scales_equals_fp8_dynamic(orc):
    M, N, K = 4, 256, 512
    Aq, _, Wq, _ = operands(orc, 2, M, N, K, seed=400)
    rng = np.random.default_rng(0)
    ra = rng.uniform(0.5, 2, M).astype(np.float32)
    rw = rng.uniform(0.5, 2, N // 128).astype(np.float32)
    sA_blk = np.repeat(ra[:, None], K // 128, axis=1)
    sW_blk = np.repeat(rw[:, None], K // 128, axis=1)
    _, ref_b, _ = orc.gemm(2, Aq, sA_blk, Wq, sW_blk)
    _, ref_d, _ = orc.gemm(0, Aq, ra, Wq, np.repeat(rw, 128))
    assert np.allclose(ref_b, ref_d, rtol=1e-14, atol=0)


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_bruteforce_tiny(orc, fmt):
    rng = np.random.default_rng(fmt)
    for M, N, K in itertools.product([1, 2, 4], [1, 3], [1, 4, 128 if fmt == 2 else 3]):
        if fmt == 1:
            Aq = rng.integers(-127, 128, (M, K)).astype(np.int8)
            Wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
            val = lambda c: float(np.int8(c))
        else:
            Aq = rng.integers(0, 256, (M, K)).astype(np.uint8)
            Wq = rng.integers(0, 256, (N, K)).astype(np.uint8)
            Aq[(Aq & 0x7F) == 0x7F] = 0x11
            Wq[(Wq & 0x7F) == 0x7F] = 0x22
            tab = decode_fp8(np.arange(256, dtype=np.uint8))
            val = lambda c: float(tab[int(c)])
        if fmt == 2:
            nbk = (K + 127) // 128
            sA = rng.uniform(0.5, 2, (M, nbk)).astype(np.float32)
            sW = rng.uniform(0.5, 2, ((N + 127) // 128, nbk)).astype(np.float32)
        else:
            sA = rng.uniform(0.5, 2, M).astype(np.float32)
            sW = rng.uniform(0.5, 2, N).astype(np.float32)
        _, ref, _ = orc.gemm(fmt, Aq, sA, Wq, sW)
        for m in range(M):
            for n in range(N):
                if fmt == 2:
                    tot = 0.0
                    for kb in range((K + 127) // 128):
                        s = 0.0
                        for k in range(kb * 128, min(K, kb * 128 + 128)):
                            s += val(Aq[m, k]) * val(Wq[n, k])
                        tot += float(sA[m, kb]) * float(sW[n // 128, kb]) * s
                else:
                    s = 0.0
                    for k in range(K):
                        s += val(Aq[m, k]) * val(Wq[n, k])
                    tot = s * float(sA[m]) * float(sW[n])
                assert abs(ref[m, n] - tot) <= 1e-12 * max(1.0, abs(tot)), (M, N, K, m, n)


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_swap_ab_identity(orc, fmt):
    M, N, K = 7, 300, 512
    Aq, sA, Wq, sW = operands(orc, fmt, M, N, K, seed=500 + fmt)
    _, ref, _ = orc.gemm(fmt, Aq, sA, Wq, sW)
    assert np.array_equal(orc.gemm_swap_ab(fmt, Aq, sA, Wq, sW), ref)


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_split_k_identity(orc, fmt):
    M, N, K = 3, 130, 1024
    Aq, sA, Wq, sW = operands(orc, fmt, M, N, K, seed=600 + fmt)
    _, ref, _ = orc.gemm(fmt, Aq, sA, Wq, sW)
    units = K // 128 if fmt == 2 else K
    for S in [1, 2, 4, 8, 16, 32, 64, 128, 256]:
        if S > units:
            continue
        r = orc.gemm_split_k(fmt, Aq, sA, Wq, sW, S)
        if fmt == 1:
            assert np.array_equal(r, ref), S
        else:
            assert np.allclose(r, ref, rtol=1e-12, atol=0), S


def test_points_match_full(orc):
    M, N, K = 5, 260, 1024
    for fmt in (0, 1, 2):
        Aq, sA, Wq, sW = operands(orc, fmt, M, N, K, seed=700 + fmt)
        _, ref, _ = orc.gemm(fmt, Aq, sA, Wq, sW)
        pm = np.array([0, 4, 2, 3]); pn = np.array([0, 259, 128, 77])
        pts = orc.gemm_points(fmt, Aq, sA, Wq, sW, pm, pn)
        assert np.allclose(pts, ref[pm, pn], rtol=1e-14, atol=0)


def test_column_slice_matches_full(orc):
    Aq, sA, Wq, sW = operands(orc, 0, 3, 300, 256, seed=800)
    out, ref, _ = orc.gemm(0, Aq, sA, Wq, sW)
    out2, ref2, _ = orc.gemm(0, Aq, sA, Wq, sW, n_lo=100, n_hi=229)
    assert np.array_equal(ref[:, 100:229], ref2) and np.array_equal(out[:, 100:229], out2)


@pytest.mark.parametrize("fmt,M,N,K", [(0, 5, 300, 640), (1, 7, 260, 1040), (2, 3, 384, 768), (0, 33, 129, 4096),
                                       (2, 9, 200, 1280)])
def test_matmul_reference_equals_the_loop(orc, fmt, M, N, K):
    """gemm_ref_matmul (numpy's matmul over the oracle's decoded codes, for full-size
    checks) gives orc_gemm's fp64 reference bit for bit: the sums of products are exact
    in fp64 at these sizes and the scales are applied in the same order."""
    x = synth.activations(M, K, seed=600 + fmt)
    w = synth.weights(N, K, seed=601 + fmt)
    if fmt == 2:
        Aq, sA = orc.quant_rows(0, synth.bf16_bits(x), group=128)
        Wq, sW = orc.quant_weight_block(synth.bf16_bits(w))
    else:
        Aq, sA = orc.quant_rows(fmt, synth.bf16_bits(x))
        Wq, sW = orc.quant_rows(fmt, synth.bf16_bits(w))
    _, ref, _ = orc.gemm(fmt, Aq, sA, Wq, sW)
    assert np.array_equal(orc.gemm_ref_matmul(fmt, Aq, sA, Wq, sW), ref)
