"""Pins of the oracle's number formats (e4m3, int8, bf16, scales) against things other
than the oracle itself: the OCP e4m3 definition table (golden anchors), torch's own
float8_e4m3fn / bfloat16 casts, torch.round, and a brute-force nearest-value search."""
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def all_bf16_floats():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = (bits.astype(np.uint32) << 16).view(np.float32)
    return f[np.isfinite(f)]


def e4m3_table():
    """Values of all 256 codes via torch's float8_e4m3fn -> float conversion."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def nearest_e4m3(v):
    """Brute-force e4m3 encode: nearest of the finite codes, ties to the even code
    (even mantissa = even code), magnitudes past 448 saturate, sign kept on zero."""
    tab = e4m3_table()
    finite = [c for c in range(256) if np.isfinite(tab[c])]
    out = np.zeros(len(v), dtype=np.uint8)
    pos = np.array([c for c in finite if c < 0x80], dtype=np.int64)   # 0x00..0x7E
    pv = tab[pos]
    for i, x in enumerate(np.asarray(v, dtype=np.float64)):
        a = abs(x)
        if a >= 448.0:
            c = 0x7E
        else:
            d = np.abs(pv - a)
            best = np.min(d)
            cands = pos[d == best]
            c = int(cands[0]) if len(cands) == 1 else int([cc for cc in cands if cc % 2 == 0][0])
        if math.copysign(1.0, x) < 0:
            c |= 0x80
        out[i] = c
    return out


def test_e4m3_golden_anchors(orc):
    with open(os.path.join(GOLDEN, "e4m3_anchors.txt")) as fh:
        rows = [ln.split() for ln in fh if ln.strip() and not ln.startswith("#")]
    for code, val in rows:
        c = int(code, 16)
        got = orc.e4m3_decode([c])[0]
        if val == "nan":
            assert np.isnan(got)
        else:
            want = float(val)
            assert got == want and math.copysign(1, got) == math.copysign(1, want), (code, got, want)
            assert orc.e4m3_encode([np.float32(want)])[0] == c


def test_e4m3_decode_matches_torch(orc):
    tab = e4m3_table()
    got = orc.e4m3_decode(np.arange(256))
    nan = np.isnan(tab)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], tab[~nan])
    assert nan.sum() == 2  # 0x7F and 0xFF


def test_e4m3_encode_all_bf16_bruteforce(orc):
    v = all_bf16_floats()
    got = orc.e4m3_encode(v)
    want = nearest_e4m3(v)
    bad = np.nonzero(got != want)[0]
    assert len(bad) == 0, [(float(v[i]), int(got[i]), int(want[i])) for i in bad[:10]]


def test_e4m3_encode_midpoints(orc):
    """At, just below and just above every midpoint between adjacent codes."""
    tab = e4m3_table()
    pos = np.sort(tab[np.isfinite(tab) & (tab >= 0)])
    pos = np.unique(pos)
    mids = (pos[:-1] + pos[1:]) / 2.0
    pts = []
    for m in mids:
        f = np.float32(m)
        assert float(f) == m  # midpoints of e4m3 values are fp32-exact
        pts += [f, np.nextafter(f, np.float32(0)), np.nextafter(f, np.float32(1e9))]
    pts = np.array(pts, dtype=np.float32)
    pts = np.concatenate([pts, -pts, np.float32([448.0, 464.0, 479.99, 480.0, 1e30, -1e30])])
    assert np.array_equal(orc.e4m3_encode(pts), nearest_e4m3(pts))


def test_e4m3_encode_matches_torch_in_range(orc):
    rng = np.random.default_rng(7)
    v = np.concatenate([all_bf16_floats(),
                        rng.standard_normal(20000).astype(np.float32) * 100,
                        rng.standard_normal(20000).astype(np.float32) * 1e-3]).astype(np.float32)
    v = v[np.abs(v) <= 448.0]
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = orc.e4m3_encode(v)
    assert np.array_equal(got, want)


def test_e4m3_nan(orc):
    assert orc.e4m3_encode([np.float32("nan")])[0] == 0x7F


def test_int8_encode_matches_torch_round(orc):
    v = np.concatenate([all_bf16_floats()[::3],
                        np.arange(-140, 140, 0.25, dtype=np.float32),
                        np.float32([0.5, 1.5, 2.5, -0.5, -2.5, 126.5, -126.5, 127.5, -127.5, 1e9, -1e9])])
    v = v.astype(np.float32)
    want = torch.clamp(torch.round(torch.from_numpy(v)), -127, 127).to(torch.int8).numpy()
    assert np.array_equal(orc.int8_encode(v), want)


def test_bf16_from_double_single_rounding(orc):
    """fp32-exact inputs: torch's fp32 -> bf16 cast (one RNE rounding) agrees.
    Doubles just off a bf16 midpoint: the result must go to the nearer side, which a
    detour through fp32 (double rounding) would get wrong."""
    rng = np.random.default_rng(3)
    f = np.concatenate([rng.standard_normal(5000).astype(np.float32) * 37,
                        rng.standard_normal(5000).astype(np.float32) * 1e-38]).astype(np.float32)
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.bf16_from_double(f.astype(np.float64)), want)
    # midpoint between bf16 1.0 and 1.0078125 is 1.00390625; nudge by 2^-40
    lo = orc.bf16_from_double([1.00390625 - 2.0 ** -40])[0]
    hi = orc.bf16_from_double([1.00390625 + 2.0 ** -40])[0]
    tie = orc.bf16_from_double([1.00390625])[0]
    assert lo == 0x3F80 and hi == 0x3F81 and tie == 0x3F80


def test_scale_fp8_int8_and_zero(orc):
    assert orc.scale(448.0, 448.0) == np.float32(1.0)
    assert orc.scale(0.0, 448.0) == np.float32(1.0)
    a = np.float32(3.7)
    assert orc.scale(a, 127.0) == np.float32(a) / np.float32(127.0)


@pytest.mark.parametrize("amax", [1e-30, 3e-5, 0.01, 1.0, 3.5, 448.0, 448.0 * 8, 1e20, 7.0 * 448])
def test_scale_ue8m0_is_smallest_power_of_two(orc, amax):
    s = float(orc.scale(np.float32(amax), 448.0, ue8m0=True))
    r = float(np.float32(amax) / np.float32(448.0))
    m, e = math.frexp(s)
    assert m == 0.5, "not a power of two"
    assert s >= r and s / 2 < r
