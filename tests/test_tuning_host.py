"""Host-side checks of the variant table and the sweep that writes it (no device: the
planner runs on the host): every shipped table entry is a legal variant for its own
shape and token bucket, and the sweep proposes only legal candidates, its reference
variant among them."""
import os

import pytest

from bit_quantized_gemm_token_b200 import sweep, w8


def table_rows():
    rows = []
    with open(w8.DEFAULT_TABLE) as fh:
        for ln in fh:
            ln = ln.split("#", 1)[0].strip()
            if ln:
                f, n, k, m, v = ln.split()
                rows.append((int(f), int(n), int(k), int(m), int(v, 16)))
    return rows


@pytest.mark.skipif(not os.path.exists(w8.DEFAULT_TABLE), reason="no shipped table")
def test_shipped_table_entries_are_legal():
    rows = table_rows()
    assert rows
    for fmt, N, K, m_max, v in rows:
        assert v & w8.W8_V_EXPLICIT
        # an entry serves the token counts above the shape's next smaller bucket
        below = [r[3] for r in rows if r[:3] == (fmt, N, K) and r[3] < m_max]
        lo = max(below) + 1 if below else 1
        for M in {lo, m_max}:
            assert w8.w8_gemm_resolve_variant(fmt, M, N, K, v) == v, (fmt, N, K, M, hex(v))


def test_shipped_table_covers_the_sweep():
    rows = {(f, n, k, m) for f, n, k, m, _ in table_rows()}
    for fmt in (0, 1, 2, 3):
        shapes = sweep.BLOCK if fmt >= 2 else sweep.DENSE
        for (K, N) in shapes:
            for M in sweep.MS:
                assert (fmt, N, K, M) in rows, (fmt, N, K, M)


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("M", [1, 8, 32])
def test_sweep_candidates_are_legal(fmt, M):
    K, N = (sweep.BLOCK if fmt >= 2 else sweep.DENSE)[0]
    cands = sweep.candidates(fmt, M, N, K, quick=True)
    assert cands and len(cands) == len(set(cands))
    for v in cands:
        assert w8.w8_gemm_resolve_variant(fmt, M, N, K, v) == v
        if fmt >= 2:
            assert not w8.describe(v)["bm64"]      # the 64-row token tile is FP8 / INT8 only
    ref = sweep.default_variant(fmt, M)
    assert w8.w8_gemm_resolve_variant(fmt, M, N, K, ref) == ref


def test_mid_and_fused_families():
    """Past 64 tokens the sweep offers CTA pairs (whole tiles and K splits that fit one
    unit per pair) and the one-CTA Standard loops; the fused family offers the decode
    form with W8_V_FUSED, legal through w8_linear."""
    K, N = 12288, 4096
    cands = sweep.candidates(0, 256, N, K, families=("mid",))
    pairs = [v for v in cands if w8.describe(v)["pair"]]
    assert pairs and any(w8.describe(v)["split_k"] == 4 for v in pairs)
    assert not any(w8.describe(v)["split_k"] == 8 for v in pairs)          # 16 tiles x 8 > 74 pairs
    for v in cands:
        assert w8.w8_gemm_resolve_variant(0, 256, N, K, v) == v
    fused = sweep.candidates(0, 8, 4096, 4096, families=("fused",))
    assert fused and all(v & w8.W8_V_FUSED and v & w8.W8_V_DECODE for v in fused)
    for v in fused:
        assert w8.w8_linear_resolve(0, 8, 4096, 4096, v) == v
    assert sweep.candidates(2, 8, 4096, 5120, families=("fused",)) == []  # no fused decode for Block-FP8
