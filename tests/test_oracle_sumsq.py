"""Pins of the oracle's sum of squares (the first step of rms_norm, "PyTorch integra
Helion en vLLM para acelerar inferencia FP8", section "Patron de fusion del forward
pass"): the exact sum of the squared bf16 values, rounded once to fp32 with ties to
even.  The reference here is written independently with Python's exact rationals
(fractions.Fraction) and integer arithmetic; the cases include rows whose exact sum
lies on, or a hair away from, an fp32 rounding midpoint -- where an fp64 running sum
would round the wrong way -- the subnormal range, overflow and special values."""
import math
from fractions import Fraction

import numpy as np
import pytest

from bit_quantized_gemm_token_b200 import synth


def bf16_bits_of(vals):
    """bf16 bit patterns of values that are exactly representable in bf16."""
    f = np.asarray(vals, dtype=np.float32)
    b = f.view(np.uint32)
    assert np.all((b & 0xFFFF) == 0), "value not representable in bf16"
    return (b >> 16).astype(np.uint16)


def exact_value(bits):
    """Exact rational value of a bf16 bit pattern (finite)."""
    b = int(bits)
    sign = -1 if b & 0x8000 else 1
    E, m = (b >> 7) & 0xFF, b & 0x7F
    if E == 0:
        return sign * Fraction(m, 1) * Fraction(1, 2 ** 133)
    return sign * Fraction(128 + m) * Fraction(2) ** (E - 134)


def round_f32(v):
    """Round a non-negative rational to fp32, nearest, ties to even (inf past the top)."""
    if v == 0:
        return np.float32(0.0)
    e = math.floor(math.log2(v.numerator) - math.log2(v.denominator))
    # fix up floating-point error in the exponent estimate
    while Fraction(2) ** e > v:
        e -= 1
    while Fraction(2) ** (e + 1) <= v:
        e += 1
    ulp = Fraction(2) ** (max(e, -126) - 23)
    q = v / ulp
    n = q.numerator // q.denominator
    r = q - n
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
        n += 1
    out = n * ulp
    if out >= Fraction(2) ** 128:
        return np.float32(np.inf)
    return np.float32(float(out))      # exactly representable: no second rounding


def ref_sumsq(bits):
    return round_f32(sum(exact_value(b) ** 2 for b in bits))


def test_random_rows(orc):
    for seed in range(6):
        x = synth.activations(3, 512, seed=500 + seed)
        bits = synth.bf16_bits(x)
        for row in bits:
            assert orc.sumsq_f32(row) == ref_sumsq(row)


def test_wide_dynamic_range(orc):
    # magnitudes from 2^-120 to 2^60 in one row: no fp64 running sum is exact here
    rng = np.random.default_rng(7)
    for _ in range(20):
        ex = rng.integers(-120, 60, size=300)
        mant = rng.integers(128, 256, size=300)
        vals = mant.astype(np.float64) * np.exp2(ex - 7)
        bits = bf16_bits_of(vals.astype(np.float32))
        assert orc.sumsq_f32(bits) == ref_sumsq(bits)


def test_midpoint_rows(orc):
    # 1 + (2^-12)^2 = 1 + 2^-24 is exactly the midpoint between 1 and the next fp32
    one, t = 1.0, 2.0 ** -12
    assert orc.sumsq_f32(bf16_bits_of([one, t])) == np.float32(1.0)            # tie: to even
    up = np.nextafter(np.float32(1.0), np.float32(2.0))
    # a tiny extra square far below fp64's resolution decides the tie upward; an fp64
    # running sum (1 + 2^-24 + 2^-100 == 1 + 2^-24) would round it to even, i.e. down
    assert orc.sumsq_f32(bf16_bits_of([one, t, 2.0 ** -50])) == up
    assert orc.sumsq_f32(bf16_bits_of([2.0 ** -50, t, one])) == up            # order-free
    # just below the midpoint: 1 + 2^-24 - tiny is impossible with squares, so use
    # (1 + 2^-7)^2 = 1 + 2^-6 + 2^-14 and pieces around its neighbours instead
    a = 1.0 + 2.0 ** -7
    base = [a, 2.0 ** -12, 2.0 ** -40]
    bits = bf16_bits_of(base)
    assert orc.sumsq_f32(bits) == ref_sumsq(bits)


def test_many_tiny_terms_cross_a_midpoint(orc):
    # 4096 squares of 2^-18 (each 2^-36) add to exactly 2^-24: with 1.0 they form a tie;
    # one more tiny term pushes it over
    bits = bf16_bits_of([1.0] + [2.0 ** -18] * 4096)
    assert orc.sumsq_f32(bits) == np.float32(1.0)
    bits2 = bf16_bits_of([1.0] + [2.0 ** -18] * 4096 + [2.0 ** -100])
    assert orc.sumsq_f32(bits2) == np.nextafter(np.float32(1.0), np.float32(2.0))
    assert orc.sumsq_f32(bits2[::-1].copy()) == orc.sumsq_f32(bits2)


def test_subnormal_and_special(orc):
    assert orc.sumsq_f32(np.zeros(8, np.uint16)) == np.float32(0.0)
    # smallest bf16 subnormal 2^-133: its square 2^-266 rounds to 0 in fp32
    assert orc.sumsq_f32(np.array([1, 1], np.uint16)) == np.float32(0.0)
    # 2^-75 squared = 2^-150: exactly half the smallest fp32 subnormal -> ties to 0;
    # two of them make 2^-149, the smallest subnormal; three round to 2^-148 (tie to even)
    h = bf16_bits_of([2.0 ** -75])
    assert orc.sumsq_f32(np.repeat(h, 1)) == np.float32(0.0)
    assert orc.sumsq_f32(np.repeat(h, 2)) == np.float32(2.0 ** -149)
    assert orc.sumsq_f32(np.repeat(h, 3)) == np.float32(2.0 ** -148)
    # (1.21875 * 2^-75)^2 = 0.7427 * 2^-149 rounds to 2^-149; rounding first to a grid
    # one bit finer (1.4854 * 2^-150 -> 2^-150) and then to fp32 would tie down to 0
    lone = bf16_bits_of([1.21875 * 2.0 ** -75])
    assert orc.sumsq_f32(lone) == np.float32(2.0 ** -149) == ref_sumsq(lone)
    rng = np.random.default_rng(3)
    for _ in range(20):
        bits = rng.integers(1, 0x0400, size=64).astype(np.uint16)   # tiny subnormal-range squares
        assert orc.sumsq_f32(bits) == ref_sumsq(bits)
    # overflow to +inf, and the non-finite inputs
    big = bf16_bits_of([2.0 ** 64, 2.0 ** 64])
    assert orc.sumsq_f32(big) == np.float32(np.inf)
    near = bf16_bits_of([1.9921875 * 2.0 ** 63])          # square just below FLT_MAX
    assert orc.sumsq_f32(near) == ref_sumsq(near) and np.isfinite(orc.sumsq_f32(near))
    assert np.isinf(orc.sumsq_f32(np.array([0x7F80, 0x3F80], np.uint16)))
    assert np.isnan(orc.sumsq_f32(np.array([0x7FC0, 0x3F80], np.uint16)))


def test_sign_is_ignored(orc):
    x = synth.bf16_bits(synth.activations(1, 256, seed=42))[0]
    assert orc.sumsq_f32(x) == orc.sumsq_f32(x ^ np.uint16(0x8000))


@pytest.mark.parametrize("H", [4096, 12288])
def test_config_rows_match_fp64_when_exact(orc, H):
    # on the workload's rows the fp64 sum of squares is usually exact; where it is (an
    # fp64 re-summation in the opposite order agrees and the fp32 rounding is away from
    # a midpoint) the oracle must give that value
    x = synth.bf16_bits(synth.activations(8, H, seed=11))
    for row in x:
        v = row.view(np.uint16).astype(np.uint32) << 16
        f = v.view(np.float32).astype(np.float64)
        s1 = float(np.sum(f * f))
        assert orc.sumsq_f32(row) == np.float32(s1) or ref_sumsq(row) == orc.sumsq_f32(row)
