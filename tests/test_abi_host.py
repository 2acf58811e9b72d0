"""Host-only checks of the C ABI: the library builds and loads, exports every entry
point include/w8.h declares, and rejects bad arguments with the documented status
codes before touching a device.  No compute call runs here (no GPU needed)."""
import ctypes
import os
import re

import pytest

from bit_quantized_gemm_token_b200 import build, w8

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return w8.lib()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "w8.h")).read()
    return re.findall(r"W8_API\s+[\w\s\*]+?\b(w8_\w+)\s*\(", src)


def test_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code in range(0, -9, -1):
        s = w8.status_string(code)
        assert s and s != "unknown status", code
    assert w8.status_string(-99) == "unknown status"
    assert w8.w8_version() >= 1


NULL = None


def test_bad_arguments_rejected_before_device(L):
    # null pointers / sizes
    assert L.w8_gemm(0, NULL, NULL, NULL, NULL, NULL, 1, 1, 16, 0, NULL, 0, NULL) == w8.W8_ERR_INVALID_ARG
    p16 = ctypes.c_void_p(1 << 20)           # aligned dummies: never dereferenced on these paths
    podd = ctypes.c_void_p((1 << 20) + 8)
    assert L.w8_gemm(0, p16, p16, p16, p16, p16, 0, 16, 16, 0, NULL, 0, NULL) == w8.W8_ERR_INVALID_ARG
    assert L.w8_gemm(0, podd, p16, p16, p16, p16, 1, 16, 16, 0, NULL, 0, NULL) == w8.W8_ERR_ALIGNMENT
    assert L.w8_quant_per_token(0, NULL, 1, 16, 16, p16, p16, 0, 0, NULL) == w8.W8_ERR_INVALID_ARG
    assert L.w8_quant_per_token(0, p16, 1, 12, 12, p16, p16, 0, 0, NULL) == w8.W8_ERR_ALIGNMENT
    assert L.w8_quant_per_token(5, p16, 1, 16, 16, p16, p16, 0, 0, NULL) == w8.W8_ERR_INVALID_ARG
    assert L.w8_quant_per_token(1, p16, 1, 256, 256, p16, p16, 128, 0, NULL) == w8.W8_ERR_UNSUPPORTED
    assert L.w8_quant_per_token(0, p16, 1, 256, 256, p16, p16, 64, 0, NULL) == w8.W8_ERR_UNSUPPORTED
    assert L.w8_quant_per_token(0, p16, 1, 65536, 65536, p16, p16, 0, 0, NULL) == w8.W8_ERR_UNSUPPORTED
    assert L.w8_rmsnorm_quant(p16, NULL, ctypes.c_float(1e-6), 1, 16, 16, p16, p16, NULL) == w8.W8_ERR_INVALID_ARG
    assert L.w8_silu_mul_quant(p16, 1, 16, 16, p16, p16, NULL) == w8.W8_ERR_INVALID_ARG   # ld < 2I
    assert L.w8_gemm_i32_debug(p16, p16, NULL, 1, 16, 16, 0, NULL, 0, NULL) == w8.W8_ERR_INVALID_ARG
    # quantize + GEMM: null input, row stride below K, misaligned x
    assert L.w8_linear(0, NULL, 16, p16, p16, p16, 1, 16, 16, 0, NULL, 0, NULL) == w8.W8_ERR_INVALID_ARG
    assert L.w8_linear(0, p16, 8, p16, p16, p16, 1, 16, 16, 0, NULL, 0, NULL) == w8.W8_ERR_INVALID_ARG
    assert L.w8_linear(0, podd, 16, p16, p16, p16, 1, 16, 16, 0, NULL, 0, NULL) == w8.W8_ERR_ALIGNMENT
    assert L.w8_linear_debug(0, p16, 16, p16, p16, p16, 1, 16, 16, 0, NULL, 0, NULL, NULL, NULL) == \
        w8.W8_ERR_INVALID_ARG
    # grouped GEMM: no experts, no offsets, more tokens per expert than rows is clamped but E = 0 is not
    assert L.w8_grouped_gemm(0, p16, p16, p16, p16, p16, p16, 0, 8, 16, 16, 8, 0, NULL, 0, NULL) == \
        w8.W8_ERR_INVALID_ARG
    assert L.w8_grouped_gemm(0, p16, p16, p16, p16, p16, NULL, 2, 8, 16, 16, 8, 0, NULL, 0, NULL) == \
        w8.W8_ERR_INVALID_ARG
    # query/key norm + rotary: head size 96 is not supported, misaligned qkv
    assert L.w8_qk_norm_rope(p16, p16, 1, 2, 1, 96, p16, p16, p16, 8, p16, ctypes.c_float(1e-6), NULL) == \
        w8.W8_ERR_UNSUPPORTED
    assert L.w8_qk_norm_rope(ctypes.c_void_p((1 << 20) + 2), p16, 1, 2, 1, 128, p16, p16, p16, 8, p16,
                             ctypes.c_float(1e-6), NULL) == w8.W8_ERR_ALIGNMENT
    assert L.w8_qk_norm_rope(p16, p16, 1, 2, 1, 128, p16, p16, ctypes.c_void_p((1 << 20) + 8), 8, p16,
                             ctypes.c_float(1e-6), NULL) == w8.W8_ERR_ALIGNMENT   # cos/sin table 16-byte
    assert L.w8_qk_norm_rope(NULL, p16, 1, 2, 1, 128, p16, p16, p16, 8, p16, ctypes.c_float(1e-6), NULL) == \
        w8.W8_ERR_INVALID_ARG


def test_valid_call_without_device_reports_no_device(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    p16 = ctypes.c_void_p(1 << 20)
    assert L.w8_quant_per_token(0, p16, 1, 16, 16, p16, p16, 0, 0, NULL) == w8.W8_ERR_NO_DEVICE
    assert L.w8_gemm(0, p16, p16, p16, p16, p16, 1, 128, 128, 0, NULL, 0, NULL) == w8.W8_ERR_NO_DEVICE


def test_linear_and_grouped_planning(L):
    w8.w8_clear_table()
    # w8_linear runs the quantizer and the GEMM unless the one-kernel form is asked for
    v = w8.w8_linear_resolve(0, 4, 4096, 4096)
    assert not (v & w8.W8_V_FUSED)
    vf = w8.w8_linear_resolve(0, 4, 4096, 4096, w8.variant(True, 4, 16, cluster=True) | w8.W8_V_FUSED)
    assert vf & w8.W8_V_FUSED
    assert L.w8_linear_resolve(0, 100, 4096, 4096, w8.variant(False, 1, 128) | w8.W8_V_FUSED) == w8.W8_ERR_UNSUPPORTED
    # the two-kernel workspace keeps the codes past the 256 KiB counter area
    assert w8.w8_linear_workspace_size(0, 4, 4096, 4096, w8.variant(True, 1, 16)) >= 65536 * 4 + 4 * 4096
    # grouped GEMM: counter area + one partial slot pair per CTA; Standard tiles are refused
    n = w8.w8_grouped_gemm_workspace_size(0, 64, 32, 1536, 2048, 4)
    assert n >= 65536 * 4 + 148 * 2 * 16 * 128 * 4
    assert L.w8_grouped_gemm_workspace_size(0, 64, 32, 1536, 2048, 4, w8.variant(False, 1, 128, stream=True)) == \
        ctypes.c_size_t(-1).value


def test_variant_resolution_and_workspace(L):
    w8.w8_clear_table()   # the built-in rule, not the shipped table
    # decode sizes, FP8 / INT8: the decode form on at most one wave of CTAs
    for fmt in (0, 1):
        for M in (1, 32, 64):
            d = w8.describe(w8.w8_gemm_resolve_variant(fmt, M, 4096, 4096))
            assert d["decode"] and 64 <= d["bn"] <= 256 and 1 <= d["c"] <= 8
            assert -(-4096 // d["bn"]) * d["c"] <= 148
    # Block-FP8 decode: Swap-AB with the narrow token tile, balanced partition
    d = w8.describe(w8.w8_gemm_resolve_variant(2, 1, 4096, 4096))
    assert d["swap_ab"] and d["stream"] and d["bn"] == 16
    assert w8.describe(w8.w8_gemm_resolve_variant(2, 32, 4096, 4096))["bn"] == 32
    assert not w8.describe(w8.w8_gemm_resolve_variant(0, 4096, 4096, 4096))["swap_ab"]
    # past 64 tokens: CTA pairs (FP8 / INT8); Block-FP8 keeps its tile
    assert w8.describe(w8.w8_gemm_resolve_variant(0, 4096, 4096, 4096))["pair"]
    assert w8.describe(w8.w8_gemm_resolve_variant(1, 256, 4096, 4096))["pair"]
    assert w8.describe(w8.w8_gemm_resolve_variant(0, 65, 4096, 4096))["pair"]
    assert not w8.describe(w8.w8_gemm_resolve_variant(0, 64, 4096, 4096))["pair"]
    assert not w8.describe(w8.w8_gemm_resolve_variant(2, 4096, 4096, 4096))["pair"]
    # explicit variants are validated
    assert L.w8_gemm_resolve_variant(0, 8, 256, 1024, w8.variant(True, split=4, bn=16)) > 0
    assert L.w8_gemm_resolve_variant(0, 8, 256, 256, w8.variant(True, split=4, bn=16)) == w8.W8_ERR_UNSUPPORTED  # 4 > 2 K blocks
    assert L.w8_gemm_resolve_variant(2, 8, 256, 256, w8.variant(True, bn=128)) == w8.W8_ERR_UNSUPPORTED  # block needs BN <= 64
    assert L.w8_gemm_resolve_variant(0, 8, 256, 200, 0) == w8.W8_ERR_ALIGNMENT          # K % 16
    assert L.w8_gemm_resolve_variant(2, 8, 256, 144, 0) == w8.W8_ERR_ALIGNMENT          # block K % 128
    # CTA pairs: Standard whole-tile loop with the 256 tile, FP8-dynamic / INT8 only
    pair = w8.variant(False, 1, 256, pair=True)
    for fmt in (0, 1):
        assert L.w8_gemm_resolve_variant(fmt, 4096, 4096, 4096, pair) > 0
        assert L.w8_gemm_workspace_size(fmt, 4096, 4096, 4096, pair) == 0
    # with a K split: one (tile, chunk) unit per pair, so tiles x split <= 74 pairs, and a workspace
    split4 = w8.variant(False, 4, 256, pair=True)
    assert L.w8_gemm_resolve_variant(0, 256, 4096, 12288, split4) > 0                 # 16 tiles x 4
    assert L.w8_gemm_workspace_size(0, 256, 4096, 12288, split4) == 256 * 1024 + 64 * 2 * 256 * 128 * 4
    assert L.w8_gemm_resolve_variant(0, 256, 4096, 12288, w8.variant(False, 8, 256, pair=True)) == \
        w8.W8_ERR_UNSUPPORTED                                                            # 16 x 8 > 74
    assert L.w8_gemm_resolve_variant(0, 256, 4096, 384, w8.variant(False, 4, 256, pair=True)) == \
        w8.W8_ERR_UNSUPPORTED                                                            # 4 > 3 K blocks
    for fmt, v in ((2, pair), (0, w8.variant(True, 1, 256, pair=True)), (0, w8.variant(False, 2, 256, pair=True)),
                   (0, w8.variant(False, 1, 128, pair=True)), (0, w8.variant(False, 1, 256, stream=True, pair=True)),
                   (0, w8.variant(False, 1, 256, bm64=True, pair=True))):
        # (the split 2 case: 256 tiles x 2 exceed the pairs)
        assert L.w8_gemm_resolve_variant(fmt, 4096, 4096, 4096, v) == w8.W8_ERR_UNSUPPORTED
    # parallel fixup: 64-row token tile only, no cluster, at most one CTA per SM
    assert L.w8_gemm_resolve_variant(0, 8, 4096, 4096, w8.variant(False, 1, 256, stream=True, bm64=True, pfix=True)) > 0
    assert L.w8_gemm_resolve_variant(0, 8, 4096, 4096, w8.variant(True, 1, 16, stream=True, pfix=True)) == \
        w8.W8_ERR_UNSUPPORTED
    assert L.w8_gemm_resolve_variant(0, 8, 4096, 4096, w8.variant(False, 2, 256, cluster=True, bm64=True, pfix=True)) == \
        w8.W8_ERR_UNSUPPORTED
    assert L.w8_gemm_resolve_variant(0, 8, 4096, 4096, w8.variant(False, 1, 256, stream=True, bm64=True, cps=2,
                                                                   pfix=True)) == w8.W8_ERR_UNSUPPORTED
    assert L.w8_gemm_resolve_variant(0, 8, 4096, 4096, w8.variant(False, 8, 128, bm64=True, pfix=True)) == \
        w8.W8_ERR_UNSUPPORTED                                                         # 32 tiles x 8 > 148 CTAs
    # workspace: none for whole-tile partitions, some for split / balanced
    assert w8.w8_gemm_workspace_size(0, 8, 256, 1024, w8.variant(True, split=1, bn=16)) == 0
    n = w8.w8_gemm_workspace_size(0, 8, 256, 1024, w8.variant(True, split=4, bn=16))
    ctas = 2 * 4                                  # 2 tiles x split 4
    assert n == 65536 * 4 + ctas * 2 * 16 * 128 * 4
    assert w8.w8_gemm_workspace_size(2, 8, 4096, 4096, 0) > 0     # Block-FP8 decode: balanced partition
    assert w8.w8_gemm_workspace_size(0, 8, 4096, 4096, 0) == 0    # decode form: reduced in the cluster


def test_table_parsing(L, tmp_path):
    p = tmp_path / "t.txt"
    v1 = w8.variant(True, split=2, bn=32)
    v2 = w8.variant(False, split=1, bn=128)
    p.write_text("# comment\n0 4096 4096 16 0x%x\n\n0 4096 4096 4096 0x%x  # prefill\n" % (v1, v2))
    try:
        assert w8.w8_load_table(str(p)) == 2
        assert w8.w8_gemm_resolve_variant(0, 8, 4096, 4096) == v1
        assert w8.w8_gemm_resolve_variant(0, 17, 4096, 4096) == v2
        assert w8.describe(w8.w8_gemm_resolve_variant(0, 8, 4096, 6144))["decode"]   # not in table: built-in rule
        bad = tmp_path / "bad.txt"
        bad.write_text("0 4096 4096 16\n")
        assert L.w8_load_table(os.fsencode(str(bad))) == w8.W8_ERR_IO
        assert L.w8_load_table(b"/nonexistent/table.txt") == w8.W8_ERR_IO
        assert w8.w8_gemm_resolve_variant(0, 8, 4096, 4096) == v1   # failed load keeps the old table
    finally:
        w8.w8_clear_table()
    assert w8.w8_gemm_resolve_variant(0, 8, 4096, 4096) != v1
    if os.path.exists(w8.DEFAULT_TABLE):
        assert w8.w8_load_table(w8.DEFAULT_TABLE) > 0
