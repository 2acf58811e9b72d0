"""The binding's constants are the header's: every numeric #define of include/w8.h that
the binding also names has the same value, and the variant helpers round-trip."""
import os
import re

import pytest

from bit_quantized_gemm_token_b200 import w8

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_defines():
    out = {}
    text = open(os.path.join(ROOT, "include", "w8.h")).read()
    for name, expr in re.findall(r"^#define\s+(W8_\w+)\s+(.+?)\s*(?:/\*.*)?$", text, flags=re.M):
        expr = expr.strip()
        shift = re.fullmatch(r"\(\s*1\s*<<\s*(\d+)\s*\)", expr)
        if shift:
            out[name] = 1 << int(shift.group(1))
        elif re.fullmatch(r"\(?-?\d+\)?", expr):
            out[name] = int(expr.strip("()"))
    return out


def test_constants_match_the_header():
    d = header_defines()
    assert len(d) >= 30
    shared = [n for n in d if hasattr(w8, n)]
    assert len(shared) >= 30
    for n in shared:
        assert getattr(w8, n) == d[n], n


@pytest.mark.parametrize("kw", [
    dict(swap=True, split=4, bn=16, cluster=True),
    dict(swap=True, split=1, bn=32, stream=True, pdl=True, stages=3, kps=2, cps=2),
    dict(swap=False, split=2, bn=256, bm64=True, pfix=True, kps=1, stages=5),
    dict(swap=False, split=1, bn=256, pair=True, stages=5, pdl=True),
    dict(swap=False, split=256, bn=128),
])
def test_variant_round_trip(kw):
    v = w8.variant(**kw)
    d = w8.describe(v)
    assert d["swap_ab"] == kw["swap"] and d["split_k"] == kw["split"] and d["bn"] == kw["bn"]
    for key in ("stream", "pdl", "cluster", "bm64", "pfix", "pair"):
        assert d[key] == kw.get(key, False), key
    for key in ("stages", "kps", "cps"):
        assert d[key] == kw.get(key, 0), key


def test_variant_rejects_non_power_of_two_split():
    with pytest.raises(ValueError):
        w8.variant(True, 3, 16)


@pytest.mark.parametrize("kw", [dict(bn=256, c=8), dict(bn=176, c=3, stages=2, l2ahead=6, pdl=True), dict(bn=64, c=1)])
def test_decode_variant_round_trip(kw):
    v = w8.decode_variant(**kw)
    d = w8.describe(v)
    assert d["decode"] and d["bn"] == kw["bn"] and d["c"] == kw["c"]
    assert d["stages"] == kw.get("stages", 0) and d["l2ahead"] == kw.get("l2ahead", 4) and d["pdl"] == kw.get("pdl", False)


def test_decode_variant_legality_without_a_device():
    # planning needs no GPU: more than 64 tokens, more chunks than K blocks and the
    # block formats are refused; a legal word resolves to itself
    v = w8.decode_variant(256, 8)
    assert w8.w8_gemm_resolve_variant(0, 16, 4096, 4096, v) == v
    for fmt, M, N, K in [(0, 65, 1024, 1024), (1, 8, 1024, 256), (2, 8, 1024, 1024)]:
        with pytest.raises(w8.W8Error):
            w8.w8_gemm_resolve_variant(fmt, M, N, K, w8.decode_variant(256, 3 if K == 256 else 1))
    with pytest.raises(ValueError):
        w8.decode_variant(200, 1)
