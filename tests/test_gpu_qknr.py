"""GPU parity of w8_qk_norm_rope (query/key rms_norm + rotary embedding) with the CPU
oracle: bf16 outputs bit for bit, in place and out of place, at decode and prefill
token counts, every supported head size; a position outside the table is reported in
the device status word."""
import numpy as np
import pytest
import torch

from bit_quantized_gemm_token_b200 import synth, w8

pytestmark = pytest.mark.gpu


def case(T, Hq, Hkv, D, seed, max_pos=4096, random_angles=True):
    qkv = synth.activations(T, (Hq + 2 * Hkv) * D, seed=seed)
    qw = synth.gamma(D, seed=seed + 1)
    kw = synth.gamma(D, seed=seed + 2)
    pos = synth.positions(T, max_pos, seed=seed + 3)
    table = synth.rope_table(max_pos, D, seed=seed + 4) if random_angles else synth.rope_table(max_pos, D, base=1e6)
    return qkv, qw, kw, pos, table


def oracle_out(orc, qkv, qw, kw, pos, table, Hq, Hkv, D):
    return orc.qk_norm_rope(synth.bf16_bits(qkv), Hq, Hkv, D, synth.bf16_bits(qw), synth.bf16_bits(kw),
                            table.numpy(), pos.numpy())


@pytest.mark.parametrize("T", [1, 3, 32, 257])
@pytest.mark.parametrize("Hq,Hkv,D", [(32, 8, 128), (16, 4, 64), (8, 2, 256), (5, 1, 128)])
@pytest.mark.parametrize("inplace", [False, True])
def test_bit_exact(orc, T, Hq, Hkv, D, inplace):
    qkv, qw, kw, pos, table = case(T, Hq, Hkv, D, seed=100 + T + D + Hq, random_angles=(T % 2 == 1))
    want = oracle_out(orc, qkv, qw, kw, pos, table, Hq, Hkv, D)
    x = qkv.cuda()
    out = x if inplace else None
    got = w8.w8_qk_norm_rope(x, Hq, Hkv, D, qw.cuda(), kw.cuda(), table.cuda(), pos.cuda(), out=out)
    torch.cuda.synchronize()
    assert np.array_equal(synth.bf16_bits(got.cpu()), want)
    assert w8.w8_device_status(clear=True) == 0


def test_prefill_qwen3_shape(orc):
    """Prefill-sized call on the usual rotary table (base 1e6), Qwen3-like heads."""
    T, Hq, Hkv, D = 4096, 32, 8, 128
    qkv, qw, kw, pos, table = case(T, Hq, Hkv, D, seed=7, max_pos=8192, random_angles=False)
    got = w8.w8_qk_norm_rope(qkv.cuda(), Hq, Hkv, D, qw.cuda(), kw.cuda(), table.cuda(), pos.cuda())
    torch.cuda.synchronize()
    rows = np.r_[0:5, 2000:2003, T - 3:T]
    want = oracle_out(orc, qkv[rows], qw, kw, pos[rows], table, Hq, Hkv, D)
    assert np.array_equal(synth.bf16_bits(got.cpu()[rows]), want)


def test_position_outside_table_reported(orc):
    T, Hq, Hkv, D = 4, 4, 2, 64
    qkv, qw, kw, pos, table = case(T, Hq, Hkv, D, seed=9, max_pos=16)
    pos[1] = 16
    w8.w8_device_status(clear=True)
    w8.w8_qk_norm_rope(qkv.cuda(), Hq, Hkv, D, qw.cuda(), kw.cuda(), table.cuda(), pos.cuda())
    torch.cuda.synchronize()
    assert w8.w8_device_status(clear=True) == w8.W8_ERR_INVALID_ARG
    assert w8.w8_device_status() == 0


def test_bad_sizes_rejected():
    x = torch.zeros((2, 4 * 96), dtype=torch.bfloat16, device="cuda")
    w = torch.ones(96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w8.W8Error) as e:
        w8.w8_qk_norm_rope(x, 2, 1, 96, w, w, torch.zeros((4, 96), device="cuda"),
                           torch.zeros(2, dtype=torch.int64, device="cuda"))
    assert e.value.code == w8.W8_ERR_UNSUPPORTED


def test_heads_on_fp32_midpoints(orc):
    """Heads whose exact sum of squares lies on or a hair past an fp32 rounding midpoint
    (1 + 2^-24) sit beside ordinary heads in the same warp: the heads whose fp64 sum
    cannot settle the rounding recompute it with double-doubles while their neighbours
    do not, and every output still equals the oracle's."""
    T, Hq, Hkv, D = 6, 8, 2, 128
    qkv, qw, kw, pos, table = case(T, Hq, Hkv, D, seed=77)
    x = qkv.float().view(T, Hq + 2 * Hkv, D)
    for t in range(T):
        for h in range(t % 3, Hq + Hkv, 3):
            x[t, h] = 0.0
            x[t, h, 0] = 1.0
            x[t, h, 5] = 2.0 ** -12
            if (t + h) % 2:
                x[t, h, D - 1] = 2.0 ** -50
    qkv = x.view(T, -1).to(torch.bfloat16)
    want = oracle_out(orc, qkv, qw, kw, pos, table, Hq, Hkv, D)
    for inplace in (False, True):
        xd = qkv.cuda()
        got = w8.w8_qk_norm_rope(xd, Hq, Hkv, D, qw.cuda(), kw.cuda(), table.cuda(), pos.cuda(),
                                 out=xd if inplace else None)
        torch.cuda.synchronize()
        assert np.array_equal(synth.bf16_bits(got.cpu()), want), inplace
    assert w8.w8_device_status(clear=True) == 0
