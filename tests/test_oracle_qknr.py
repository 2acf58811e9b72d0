"""Pins of the oracle's query/key rms_norm + rotary embedding against things other than
itself: at a zero angle it is torch's rms_norm per head; the rotation is a complex
multiplication of each (i, i + D/2) pair; rotations keep the pair's length; the table
row follows the token's position; value heads pass through untouched."""
import numpy as np
import pytest
import torch

from bit_quantized_gemm_token_b200 import synth

T, HQ, HKV, D = 5, 4, 2, 128
H = HQ + 2 * HKV


def inputs(seed=7, max_pos=64):
    qkv = synth.activations(T, H * D, seed=seed)
    qw = synth.gamma(D, seed=seed + 1)
    kw = synth.gamma(D, seed=seed + 2)
    pos = synth.positions(T, max_pos, seed=seed + 3)
    return qkv, qw, kw, pos


def bf(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double()


def ref_norm(qkv, qw, kw, eps=1e-6):
    """torch's rms_norm per query / key head, in fp64, of the bf16 inputs."""
    x = qkv.double().view(T, H, D)
    q = torch.nn.functional.rms_norm(x[:, :HQ], (D,), weight=qw.double(), eps=eps)
    k = torch.nn.functional.rms_norm(x[:, HQ:HQ + HKV], (D,), weight=kw.double(), eps=eps)
    return q, k


def run(orc, qkv, qw, kw, table, pos):
    out = orc.qk_norm_rope(synth.bf16_bits(qkv), HQ, HKV, D, synth.bf16_bits(qw), synth.bf16_bits(kw),
                           table.numpy(), pos.numpy())
    return bf(out).view(T, H, D)


def test_zero_angle_is_rms_norm_per_head(orc):
    qkv, qw, kw, pos = inputs()
    table = torch.cat([torch.ones(64, D // 2), torch.zeros(64, D // 2)], dim=1)
    got = run(orc, qkv, qw, kw, table, pos)
    q, k = ref_norm(qkv, qw, kw)
    for a, b in ((got[:, :HQ], q), (got[:, HQ:HQ + HKV], k)):
        # one bf16 rounding of the fp32 steps vs of the fp64 value
        assert torch.all((a - b).abs() <= b.abs() * 2.0 ** -8 + 1e-30)
        assert (a == b.to(torch.bfloat16).double()).double().mean() > 0.99


def test_value_heads_untouched(orc):
    qkv, qw, kw, pos = inputs(seed=11)
    got = run(orc, qkv, qw, kw, synth.rope_table(64, D, seed=3), pos)
    assert torch.equal(got[:, HQ + HKV:], qkv.double().view(T, H, D)[:, HQ + HKV:])


def test_rotation_is_complex_multiplication(orc):
    qkv, qw, kw, pos = inputs(seed=13)
    table = synth.rope_table(64, D, seed=5)
    got = run(orc, qkv, qw, kw, table, pos)
    q, k = ref_norm(qkv, qw, kw)
    c = table.double()[pos][:, None, : D // 2]
    s = table.double()[pos][:, None, D // 2:]
    for a, y in ((got[:, :HQ], q), (got[:, HQ:HQ + HKV], k)):
        z = torch.complex(y[..., : D // 2], y[..., D // 2:]) * torch.complex(c, s)
        want = torch.cat([z.real, z.imag], dim=-1)
        mag = torch.cat([z.abs(), z.abs()], dim=-1)
        assert torch.all((a - want).abs() <= mag * 2.0 ** -6 + 1e-6)


def test_rotation_keeps_pair_length(orc):
    qkv, qw, kw, pos = inputs(seed=17)
    table = synth.rope_table(64, D, seed=9)
    got = run(orc, qkv, qw, kw, table, pos)
    zero = torch.cat([torch.ones(64, D // 2), torch.zeros(64, D // 2)], dim=1)
    flat = run(orc, qkv, qw, kw, zero, pos)
    for a, b in ((got[:, :HQ + HKV], flat[:, :HQ + HKV]),):
        la = a[..., : D // 2] ** 2 + a[..., D // 2:] ** 2
        lb = b[..., : D // 2] ** 2 + b[..., D // 2:] ** 2
        assert torch.all((la - lb).abs() <= lb * 2.0 ** -5 + 1e-6)


def test_table_row_follows_position(orc):
    qkv, qw, kw, pos = inputs(seed=19)
    table = synth.rope_table(64, D, base=1e6)
    perm = torch.randperm(64, generator=torch.Generator().manual_seed(1))
    inv = torch.argsort(perm)
    a = run(orc, qkv, qw, kw, table, pos)
    b = run(orc, qkv, qw, kw, table[perm], inv[pos])      # same rows, renumbered
    assert torch.equal(a, b)
    c = run(orc, qkv, qw, kw, table, (pos + 1) % 64)
    assert not torch.equal(a[:, :HQ], c[:, :HQ])


def test_position_out_of_range_rejected(orc):
    qkv, qw, kw, pos = inputs(seed=23)
    pos[2] = 64
    with pytest.raises(ValueError):
        run(orc, qkv, qw, kw, synth.rope_table(64, D, seed=1), pos)
