"""GPU parity of the quantizers and fused producers against the CPU oracle: codes and
scales must match bit for bit."""
import numpy as np
import pytest
import torch

from bit_quantized_gemm_token_b200 import synth, w8
from gpu_helpers import bits, u8

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("qfmt", [w8.W8_Q_FP8, w8.W8_Q_INT8])
@pytest.mark.parametrize("M,K", [(1, 8), (1, 1024), (3, 4096), (16, 4096), (32, 12288), (7, 25600),
                                 (257, 1024), (2, 32768), (5, 136)])
def test_per_token_bit_exact(orc, qfmt, M, K):
    x = synth.activations(M, K, seed=1000 + M * 7 + K)
    q, s = w8.w8_quant_per_token(x.cuda(), qfmt)
    torch.cuda.synchronize()
    oq, os_ = orc.quant_rows(qfmt, bits(x))
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(u8(q), oq.view(np.uint8))


def test_per_token_strided_and_zero_rows(orc):
    M, K = 6, 1024
    big = synth.activations(M, K + 64, seed=77)
    big[2] = 0.0
    big[4, :] = -0.0
    xd = big.cuda()[:, :K]
    for qfmt in (0, 1):
        q, s = w8.w8_quant_per_token(xd, qfmt)
        oq, os_ = orc.quant_rows(qfmt, bits(big[:, :K].contiguous()))
        assert np.array_equal(s.cpu().numpy(), os_)
        assert np.array_equal(u8(q), oq.view(np.uint8))
        assert os_[2] == 1.0


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("M,K", [(1, 128), (5, 4096), (32, 5120), (17, 25600), (300, 1024)])
def test_group128_bit_exact(orc, ue8m0, M, K):
    x = synth.activations(M, K, seed=2000 + M + K)
    q, s = w8.w8_quant_per_token(x.cuda(), w8.W8_Q_FP8, group=128, ue8m0=ue8m0)
    oq, os_ = orc.quant_rows(0, bits(x), group=128, ue8m0=ue8m0)
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(u8(q), oq)


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("N,K", [(128, 128), (300, 520), (1024, 4096)])
def test_weight_block_bit_exact(orc, ue8m0, N, K):
    w = synth.weights(N, K, seed=3000 + N + K)
    q, s = w8.w8_quant_weight_block(w.cuda(), ue8m0=ue8m0)
    oq, os_ = orc.quant_weight_block(bits(w), ue8m0=ue8m0)
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(u8(q), oq)


@pytest.mark.parametrize("M,H", [(1, 4096), (5, 4096), (32, 4096), (300, 1024), (3, 8), (2, 25600)])
def test_rmsnorm_quant_bit_exact(orc, M, H):
    x = synth.activations(M, H, seed=4000 + M + H)
    g = synth.gamma(H, seed=4001 + H)
    q, s = w8.w8_rmsnorm_quant(x.cuda(), g.cuda(), 1e-6)
    oq, os_ = orc.rmsnorm_quant(bits(x), bits(g), 1e-6)
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(u8(q), oq)


@pytest.mark.parametrize("M,I", [(1, 12288), (3, 12288), (32, 12288), (64, 1024), (2, 8), (4, 25600)])
def test_silu_mul_quant_bit_exact(orc, M, I):
    xgu = synth.activations(M, 2 * I, seed=5000 + M + I)
    q, s = w8.w8_silu_mul_quant(xgu.cuda())
    oq, os_ = orc.silu_mul_quant(bits(xgu))
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(u8(q), oq)


def test_silu_mul_quant_extreme_gates(orc):
    I = 64
    g = torch.linspace(-120, 120, I).to(torch.bfloat16)
    u = torch.linspace(3, -3, I).to(torch.bfloat16)
    xgu = torch.cat([g, u])[None, :].repeat(2, 1)
    q, s = w8.w8_silu_mul_quant(xgu.cuda())
    oq, os_ = orc.silu_mul_quant(bits(xgu))
    assert np.array_equal(s.cpu().numpy(), os_) and np.array_equal(u8(q), oq)


def test_quant_prefill_rows(orc):
    """Config-5 prefill activation shape (4096 x 4096), rows checked in full."""
    M, K = 4096, 4096
    x = synth.activations(M, K, seed=6000)
    q, s = w8.w8_quant_per_token(x.cuda(), 0)
    oq, os_ = orc.quant_rows(0, bits(x))
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(u8(q), oq)


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("M,H", [(1, 4096), (5, 4096), (32, 5120), (300, 1024), (2, 25600), (3, 128)])
def test_rmsnorm_quant_group_bit_exact(orc, M, H, ue8m0):
    x = synth.activations(M, H, seed=4100 + M + H)
    g = synth.gamma(H, seed=4101 + H)
    q, s = w8.w8_rmsnorm_quant_group(x.cuda(), g.cuda(), 1e-6, 128, ue8m0)
    oq, os_ = orc.rmsnorm_quant_group(bits(x), bits(g), 1e-6, 128, ue8m0)
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(u8(q), oq)


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("M,I", [(1, 12288), (3, 12288), (32, 12288), (64, 1024), (4, 25600), (2, 128)])
def test_silu_mul_quant_group_bit_exact(orc, M, I, ue8m0):
    xgu = synth.activations(M, 2 * I, seed=5100 + M + I)
    q, s = w8.w8_silu_mul_quant_group(xgu.cuda(), 128, ue8m0)
    oq, os_ = orc.silu_mul_quant_group(bits(xgu), 128, ue8m0)
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(u8(q), oq)


def _midpoint_rows(H):
    """Rows whose exact sum of squares lies on, or a hair past, an fp32 rounding midpoint
    (1 + 2^-24 between 1 and the next fp32 value): a running fp64 sum rounds the second
    and third the wrong way."""
    rows = np.zeros((3, H), dtype=np.float32)
    rows[0, :2] = [1.0, 2.0 ** -12]                       # on the midpoint: ties to even (1)
    rows[1, :3] = [1.0, 2.0 ** -12, 2.0 ** -50]           # just past it: rounds up
    rows[2, 0] = 1.0                                      # 4096 squares of 2^-36 add to 2^-24, one more past it
    rows[2, 1:4097] = 2.0 ** -18
    rows[2, H - 1] = 2.0 ** -60
    return torch.from_numpy(rows).to(torch.bfloat16)


def test_rmsnorm_sum_of_squares_at_fp32_midpoints(orc):
    """The sum of squares is the exact sum rounded once to fp32, whatever the order the
    GPU adds in: with gamma = 1 and eps = 0 the scale is RN(RN(1 * r) / 448) with r =
    1 / sqrt(ss / H), which moves with the last bit of ss."""
    H = 8192
    x = _midpoint_rows(H)
    g = torch.ones(H, dtype=torch.bfloat16)
    q, s = w8.w8_rmsnorm_quant(x.cuda(), g.cuda(), 0.0)
    oq, os_ = orc.rmsnorm_quant(bits(x), bits(g), 0.0)
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(u8(q), oq)
    # the rows do test the rounding: an fp64 running sum would give other scales for
    # the rows past the midpoint
    xf = x.float().numpy().astype(np.float64)
    for i in (1, 2):
        naive = np.float32(np.sum(xf[i] * xf[i]))
        r = np.float32(1.0) / np.sqrt(naive / np.float32(H))
        assert np.float32(r / np.float32(448.0)) != os_[i]


def test_rmsnorm_quant_independent_of_element_order(orc):
    """Permuting a row's elements (and gamma with them) permutes the codes and leaves the
    scale alone: the sum of squares is the exact sum rounded once, so the order in which
    the GPU's threads add cannot show.  Rows with a wide spread of magnitudes (a few
    values 2^20 times the rest) make a plain fp32 sum order-dependent."""
    M, H = 16, 4096
    x = synth.activations(M, H, seed=4400).float()
    x[:, ::512] *= 2.0 ** 20
    x = x.to(torch.bfloat16)
    g = synth.gamma(H, seed=4401)
    perm = torch.from_numpy(np.random.default_rng(4402).permutation(H))
    q, s = w8.w8_rmsnorm_quant(x.cuda(), g.cuda(), 1e-6)
    qp, sp = w8.w8_rmsnorm_quant(x[:, perm].contiguous().cuda(), g[perm].contiguous().cuda(), 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(s.cpu(), sp.cpu())
    assert np.array_equal(u8(q)[:, perm.numpy()], u8(qp))
    oq, os_ = orc.rmsnorm_quant(bits(x), bits(g), 1e-6)
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(u8(q), oq)
