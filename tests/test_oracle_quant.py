"""Pins of the oracle's quantizers and fused producers.

Each check recomputes the result through a different route (torch reductions and
torch's own fp8 / round casts, fp64 numpy maths, closed forms) or checks an invariant
the definition forces (the largest element lands on +-448 / +-127, the dequantization
error stays within half a code step)."""
import math

import numpy as np
import pytest
import torch

from bit_quantized_gemm_token_b200 import synth


def torch_quant(x_f32, qfmt, group=0, ue8m0=False):
    """Independent restatement with torch primitives: amax by torch.amax, s = amax/Q in
    fp32 (1 for an all-zero group), power of two by ceil(log2) in fp64, codes by
    torch's float8_e4m3fn cast or torch.round + clamp."""
    x = torch.from_numpy(np.ascontiguousarray(x_f32, dtype=np.float32))
    M, K = x.shape
    g = K if group == 0 else group
    xg = x.reshape(M, K // g, g)
    amax = xg.abs().amax(dim=2)
    Q = 448.0 if qfmt == 0 else 127.0
    s = amax / torch.tensor(Q, dtype=torch.float32)
    if ue8m0:
        p = torch.ceil(torch.log2(s.double())).clamp(-127, 127)
        s = torch.pow(torch.tensor(2.0, dtype=torch.float64), p).float()
    s = torch.where(amax > 0, s, torch.ones_like(s))
    v = xg / s[:, :, None]
    if qfmt == 0:
        q = v.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    else:
        q = torch.clamp(torch.round(v), -127, 127).to(torch.int8)
    return q.reshape(M, K).numpy(), s.numpy()


@pytest.mark.parametrize("qfmt", [0, 1])
@pytest.mark.parametrize("M,K", [(1, 128), (5, 1024), (16, 4096), (3, 12288)])
def test_per_token_matches_torch(orc, qfmt, M, K):
    x = synth.activations(M, K, seed=11 + K + M)
    q, s = orc.quant_rows(qfmt, synth.bf16_bits(x))
    tq, ts = torch_quant(x.float().numpy(), qfmt)
    assert np.array_equal(s, ts[:, 0])
    assert np.array_equal(q.view(np.uint8), tq.view(np.uint8))


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("M,K", [(1, 128), (7, 1024), (32, 5120)])
def test_per_group_matches_torch(orc, ue8m0, M, K):
    x = synth.activations(M, K, seed=21 + K + M)
    q, s = orc.quant_rows(0, synth.bf16_bits(x), group=128, ue8m0=ue8m0)
    tq, ts = torch_quant(x.float().numpy(), 0, group=128, ue8m0=ue8m0)
    assert np.array_equal(s, ts)
    assert np.array_equal(q, tq)


@pytest.mark.parametrize("qfmt,Q,code", [(0, 448.0, 0x7E), (1, 127.0, 127)])
def test_amax_element_hits_the_top_code(orc, qfmt, Q, code):
    x = synth.activations(9, 2048, seed=5)
    xf = x.float().numpy()
    q, s = orc.quant_rows(qfmt, synth.bf16_bits(x))
    q8 = q.view(np.uint8) if qfmt == 0 else q
    for m in range(9):
        k = int(np.argmax(np.abs(xf[m])))
        if qfmt == 0:
            assert q8[m, k] & 0x7F == code and (q8[m, k] >> 7) == (xf[m, k] < 0)
        else:
            assert abs(int(q8[m, k])) == code and np.sign(q8[m, k]) == np.sign(xf[m, k])
    if qfmt == 1:
        assert np.all(np.abs(q.astype(np.int32)) <= 127)
    else:
        dec = orc.e4m3_decode(q)
        assert np.all(np.abs(dec) <= 448.0)


def test_dequant_error_within_half_step(orc):
    """|dec(q) * s - x| <= half the e4m3 spacing at x/s, times s (fp8);
    <= s/2 (int8)."""
    x = synth.activations(8, 4096, seed=9)
    xf = x.float().numpy().astype(np.float64)
    q, s = orc.quant_rows(0, synth.bf16_bits(x))
    v = xf / s[:, None]
    dec = orc.e4m3_decode(q)
    a = np.abs(v)
    step = np.where(a < 2 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(a, 1e-300))) - 3))
    assert np.all(np.abs(dec - v) <= step / 2 * (1 + 1e-6) + 1e-12)
    qi, si = orc.quant_rows(1, synth.bf16_bits(x))
    assert np.all(np.abs(qi.astype(np.float64) * si[:, None] - xf) <= si[:, None] / 2 * (1 + 1e-6))


def test_zero_row_reading(orc):
    x = torch.zeros(2, 256, dtype=torch.bfloat16)
    x[1, 3] = -0.0
    q, s = orc.quant_rows(0, synth.bf16_bits(x))
    assert np.all(s == 1.0) and np.all(q[0] == 0)
    qi, si = orc.quant_rows(1, synth.bf16_bits(x))
    assert np.all(si == 1.0) and np.all(qi == 0)


def test_weight_block_matches_torch(orc):
    N, K = 384, 512
    w = synth.weights(N, K, seed=31)
    for ue8m0 in (False, True):
        q, s = orc.quant_weight_block(synth.bf16_bits(w), ue8m0=ue8m0)
        wf = torch.from_numpy(w.float().numpy())
        blk = wf.reshape(N // 128, 128, K // 128, 128)
        amax = blk.abs().amax(dim=(1, 3))
        ts = amax / torch.tensor(448.0)
        if ue8m0:
            ts = torch.pow(torch.tensor(2.0, dtype=torch.float64), torch.ceil(torch.log2(ts.double()))).float()
        assert np.array_equal(s, ts.numpy())
        v = blk / ts[:, None, :, None]
        tq = v.to(torch.float8_e4m3fn).view(torch.uint8).reshape(N, K).numpy()
        assert np.array_equal(q, tq)


# --- rms_norm + quant -----------------------------------------------------------

def test_rmsnorm_against_fp64(orc):
    M, H = 6, 4096
    x = synth.activations(M, H, seed=41)
    g = synth.gamma(H, seed=42)
    y = orc.rmsnorm_f32(synth.bf16_bits(x), synth.bf16_bits(g), 1e-6)
    xf = x.double().numpy()
    gf = g.double().numpy()
    y64 = xf / np.sqrt(np.mean(xf * xf, axis=1, keepdims=True) + 1e-6) * gf
    rel = np.abs(y - y64) / np.maximum(np.abs(y64), 1e-30)
    assert np.max(rel) < 4 * 2.0 ** -24


def test_rmsnorm_closed_forms(orc):
    H = 1024
    ones = torch.ones(H, dtype=torch.bfloat16)
    x = torch.full((3, H), 2.0, dtype=torch.bfloat16)
    x[1] = -0.5
    x[2, ::2] = 3.0
    x[2, 1::2] = -3.0
    y = orc.rmsnorm_f32(synth.bf16_bits(x), synth.bf16_bits(ones), 0.0)
    # constant |c| rows with gamma = 1 and eps = 0 normalise to exactly +-1
    assert np.all(y[0] == 1.0) and np.all(y[1] == -1.0)
    assert np.all(np.abs(y[2]) == 1.0)
    z = orc.rmsnorm_f32(synth.bf16_bits(synth.activations(4, H, seed=3)), synth.bf16_bits(ones), 1e-6)
    rms = np.sqrt(np.mean(z.astype(np.float64) ** 2, axis=1))
    assert np.allclose(rms, 1.0, atol=1e-6)


def test_rmsnorm_quant_codes(orc):
    M, H = 5, 4096
    x = synth.activations(M, H, seed=43)
    g = synth.gamma(H, seed=44)
    q, s = orc.rmsnorm_quant(synth.bf16_bits(x), synth.bf16_bits(g), 1e-6)
    y = orc.rmsnorm_f32(synth.bf16_bits(x), synth.bf16_bits(g), 1e-6)
    tq, ts = torch_quant(y, 0)
    assert np.array_equal(s, ts[:, 0]) and np.array_equal(q, tq)


# --- exp / silu_and_mul + quant ----------------------------------------------------

def ulp32(v):
    v = np.abs(np.asarray(v, dtype=np.float32))
    return np.spacing(v).astype(np.float64)


def test_exp_within_two_ulp(orc):
    xs = np.concatenate([np.linspace(-87.0, 88.0, 40001, dtype=np.float32),
                         np.linspace(-1, 1, 20001, dtype=np.float32),
                         synth.activations(1, 5000, seed=1).float().numpy()[0]]).astype(np.float32)
    got = orc.exp_f32(xs).astype(np.float64)
    want = np.array([math.exp(float(v)) for v in xs])
    err = np.abs(got - want) / ulp32(want.astype(np.float32))
    assert np.max(err) <= 2.0, float(np.max(err))
    assert orc.exp_f32([0.0])[0] == 1.0
    assert np.isinf(orc.exp_f32([100.5])[0]) and orc.exp_f32([-160.0])[0] == 0.0
    # subnormal results stay accurate to an absolute 2^-149
    t = np.float32(-100.0)
    assert abs(float(orc.exp_f32([t])[0]) - math.exp(-100.0)) <= 2.0 ** -149


def test_silu_mul_against_fp64(orc):
    M, I = 4, 2048
    xgu = synth.activations(M, 2 * I, seed=51)
    h = orc.silu_mul_f32(synth.bf16_bits(xgu))
    xf = xgu.double().numpy()
    gte, up = xf[:, :I], xf[:, I:]
    h64 = gte / (1.0 + np.exp(-gte)) * up
    err = np.abs(h - h64) / np.maximum(ulp32(h64.astype(np.float32)), 2.0 ** -149)
    assert np.max(err) <= 4.0


def test_silu_special_values(orc):
    I = 8
    g = torch.tensor([0.0, 60.0, -60.0, 1.0, -1.0, 120.0, -120.0, 2.0], dtype=torch.bfloat16)
    u = torch.tensor([5.0, 2.0, 3.0, 1.0, 1.0, 1.0, 1.0, -4.0], dtype=torch.bfloat16)
    h = orc.silu_mul_f32(synth.bf16_bits(torch.cat([g, u])[None, :]))[0]
    assert h[0] == 0.0
    assert h[1] == 120.0                 # silu(60) = 60 in fp32
    assert abs(h[2]) < 1e-23             # silu(-60) ~ -5e-25
    assert h[5] == 120.0 and h[6] == 0.0 # exp saturates to inf / 0 cleanly
    assert abs(h[3] - 0.7310585786300049) < 1e-7
    assert abs(h[7] - (-4 * 2 / (1 + math.exp(-2)))) < 1e-5


def test_silu_mul_quant_codes(orc):
    M, I = 3, 12288
    xgu = synth.activations(M, 2 * I, seed=53)
    q, s = orc.silu_mul_quant(synth.bf16_bits(xgu))
    h = orc.silu_mul_f32(synth.bf16_bits(xgu))
    tq, ts = torch_quant(h, 0)
    assert np.array_equal(s, ts[:, 0]) and np.array_equal(q, tq)


@pytest.mark.parametrize("ue8m0", [False, True])
def test_rmsnorm_quant_group_codes(orc, ue8m0):
    M, H = 4, 4096
    x = synth.activations(M, H, seed=45)
    g = synth.gamma(H, seed=46)
    q, s = orc.rmsnorm_quant_group(synth.bf16_bits(x), synth.bf16_bits(g), 1e-6, 128, ue8m0)
    y = orc.rmsnorm_f32(synth.bf16_bits(x), synth.bf16_bits(g), 1e-6)
    tq, ts = torch_quant(y, 0, group=128, ue8m0=ue8m0)
    assert np.array_equal(s, ts) and np.array_equal(q, tq)


@pytest.mark.parametrize("ue8m0", [False, True])
def test_silu_mul_quant_group_codes(orc, ue8m0):
    M, I = 3, 12288
    xgu = synth.activations(M, 2 * I, seed=55)
    q, s = orc.silu_mul_quant_group(synth.bf16_bits(xgu), 128, ue8m0)
    h = orc.silu_mul_f32(synth.bf16_bits(xgu))
    tq, ts = torch_quant(h, 0, group=128, ue8m0=ue8m0)
    assert np.array_equal(s, ts) and np.array_equal(q, tq)
