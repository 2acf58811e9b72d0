"""Parity at the full workload sizes, in the launch configuration the benchmark times
(AUTO variant with programmatic dependent launch): the FP8-dynamic and INT8 decode
sweeps over the four dense-decoder shapes, the Block-FP8 shapes, and the fused MLP
chain (decode and prefill).  Quantized bytes and scales are compared in full; GEMM
outputs of the decode sizes in full (every row and column, against the oracle's fp64
reference formed with a matmul over its decoded codes), INT8 accumulators of every
row bit for bit; the prefill MLP sizes on whole sampled rows."""
import numpy as np
import pytest
import torch

from bit_quantized_gemm_token_b200 import synth, w8
from gpu_helpers import TOL_ABS, TOL_REL, bits, u8

pytestmark = pytest.mark.gpu

DENSE = [(4096, 6144), (4096, 4096), (4096, 24576), (12288, 4096)]      # (K, N)
BLOCK = [(5120, 10240), (5120, 51200), (25600, 5120), (4096, 6144)]
MS = [1, 2, 4, 8, 16, 32]
AUTO_PDL = w8.W8_VARIANT_AUTO | w8.W8_V_PDL


def check_full(orc, fmt, out, ops, what):
    """Every output against the oracle's fp64 reference (gemm_ref_matmul, equal to the
    oracle loop's reference bit for bit)."""
    Aq, sA, Wq, sW = ops
    ref = orc.gemm_ref_matmul(fmt, Aq, sA, Wq, sW)
    outc = out.float().cpu().double().numpy()
    assert np.all(np.isfinite(outc)), what + " non-finite output"
    err = np.max(np.abs(outc - ref))
    bound = TOL_REL * np.max(np.abs(ref)) + TOL_ABS
    assert err <= bound, "%s max err %.3g > %.3g" % (what, err, bound)


@pytest.mark.parametrize("fmt", [w8.W8_FMT_FP8_DYN, w8.W8_FMT_INT8])
@pytest.mark.parametrize("K,N", DENSE)
def test_dense_decode_sweep(orc, fmt, K, N):
    qf = w8.W8_Q_INT8 if fmt == w8.W8_FMT_INT8 else w8.W8_Q_FP8
    w = synth.weights(N, K, seed=synth.SEED_BASE + 2 + N)
    Wq_g, sW_g = w8.w8_quant_per_token(w.cuda(), qf)          # per-output-channel weights
    Wq_o, sW_o = orc.quant_rows(qf, bits(w))
    assert np.array_equal(sW_g.cpu().numpy(), sW_o) and np.array_equal(u8(Wq_g), Wq_o.view(np.uint8))
    del w
    for M in MS:
        x = synth.activations(M, K, seed=synth.SEED_BASE + 2 + M * 100 + K)
        Aq_g, sA_g = w8.w8_quant_per_token(x.cuda(), qf)
        Aq_o, sA_o = orc.quant_rows(qf, bits(x))
        assert np.array_equal(u8(Aq_g), Aq_o.view(np.uint8)) and np.array_equal(sA_g.cpu().numpy(), sA_o)
        out = w8.w8_gemm(fmt, Aq_g, sA_g, Wq_g, sW_g, variant=AUTO_PDL)
        if fmt == w8.W8_FMT_INT8:
            # every accumulator, exactly (the oracle's integer sum is numpy's int64 matmul here)
            acc = w8.w8_gemm_i32_debug(Aq_g, Wq_g, variant=AUTO_PDL)
            oacc = Aq_o.view(np.int8).astype(np.int64) @ Wq_o.view(np.int8).astype(np.int64).T
            assert np.array_equal(acc.cpu().numpy().astype(np.int64), oacc)
        torch.cuda.synchronize()
        check_full(orc, fmt, out, (Aq_o, sA_o, Wq_o, sW_o), "fmt%d %dx%d M=%d" % (fmt, K, N, M))
    assert w8.w8_device_status(clear=True) == 0


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("K,N", BLOCK)
def test_block_decode_sweep(orc, K, N, ue8m0):
    fmt = w8.W8_FMT_BLOCK_FP8_UE8M0 if ue8m0 else w8.W8_FMT_BLOCK_FP8
    w = synth.weights(N, K, seed=synth.SEED_BASE + 4 + N)
    Wq_g, sW_g = w8.w8_quant_weight_block(w.cuda(), ue8m0=ue8m0)
    Wq_o, sW_o = orc.quant_weight_block(bits(w), ue8m0=ue8m0)
    assert np.array_equal(sW_g.cpu().numpy(), sW_o) and np.array_equal(u8(Wq_g), Wq_o)
    del w
    for M in (1, 7, 32):
        x = synth.activations(M, K, seed=synth.SEED_BASE + 4 + M * 100 + K)
        Aq_g, sA_g = w8.w8_quant_per_token(x.cuda(), w8.W8_Q_FP8, group=128, ue8m0=ue8m0)
        Aq_o, sA_o = orc.quant_rows(0, bits(x), group=128, ue8m0=ue8m0)
        assert np.array_equal(u8(Aq_g), Aq_o) and np.array_equal(sA_g.cpu().numpy(), sA_o)
        out = w8.w8_gemm(fmt, Aq_g, sA_g, Wq_g, sW_g, variant=AUTO_PDL)
        torch.cuda.synchronize()
        check_full(orc, 2, out, (Aq_o, sA_o, Wq_o, sW_o), "block %dx%d M=%d" % (K, N, M))


@pytest.fixture(scope="module")
def mlp(orc):
    H, I = 4096, 12288
    g = synth.gamma(H, seed=synth.SEED_BASE + 5)
    w_gu = synth.weights(2 * I, H, seed=synth.SEED_BASE + 5 + 1)
    w_d = synth.weights(H, I, seed=synth.SEED_BASE + 5 + 2)
    gu_g = w8.w8_quant_per_token(w_gu.cuda(), 0)
    d_g = w8.w8_quant_per_token(w_d.cuda(), 0)
    gu_o = orc.quant_rows(0, bits(w_gu))
    d_o = orc.quant_rows(0, bits(w_d))
    return H, I, g, gu_g, d_g, gu_o, d_o


@pytest.mark.parametrize("M", [1, 4, 32, 256, 1024, 4096])
def test_mlp_chain(orc, mlp, M):
    """rms_norm+quant -> gate_up GEMM -> silu_and_mul+quant -> down GEMM.  Rows are
    independent, so prefill sizes are checked on a sample of whole rows."""
    H, I, g, gu_g, d_g, gu_o, d_o = mlp
    x = synth.activations(M, H, seed=synth.SEED_BASE + 5 + 10 * M)
    xd, gd = x.cuda(), g.cuda()
    q1, s1 = w8.w8_rmsnorm_quant(xd, gd, 1e-6)
    gu = w8.w8_gemm(0, q1, s1, gu_g[0], gu_g[1], variant=AUTO_PDL)
    q2, s2 = w8.w8_silu_mul_quant(gu)
    y = w8.w8_gemm(0, q2, s2, d_g[0], d_g[1], variant=AUTO_PDL)
    torch.cuda.synchronize()
    rows = list(range(M)) if M <= 4 else sorted(set(np.random.default_rng(M).integers(0, M, 6).tolist()) | {0, M - 1})
    xr = x[rows].contiguous()
    oq1, os1 = orc.rmsnorm_quant(bits(xr), bits(g), 1e-6)
    assert np.array_equal(u8(q1)[rows], oq1) and np.array_equal(s1.cpu().numpy()[rows], os1)
    gu_bits, gu_ref, _ = orc.gemm(0, oq1, os1, gu_o[0], gu_o[1])
    gu_out = gu.float().cpu().double().numpy()[rows]
    assert np.max(np.abs(gu_out - gu_ref)) <= TOL_REL * np.max(np.abs(gu_ref)) + TOL_ABS
    oq2, os2 = orc.silu_mul_quant(gu_bits)
    _, y_ref, _ = orc.gemm(0, oq2, os2, d_o[0], d_o[1])
    yo = y.float().cpu().double().numpy()[rows]
    # the chain's intermediate bf16 may differ in the last bit, which moves a few codes by
    # one step; the end-to-end bound is the GEMM bound
    assert np.max(np.abs(yo - y_ref)) <= TOL_REL * np.max(np.abs(y_ref)) + TOL_ABS


@pytest.fixture(scope="module")
def mlp_block(orc):
    H, I = 4096, 12288
    g = synth.gamma(H, seed=synth.SEED_BASE + 6)
    w_gu = synth.weights(2 * I, H, seed=synth.SEED_BASE + 6 + 1)
    w_d = synth.weights(H, I, seed=synth.SEED_BASE + 6 + 2)
    gu_g = w8.w8_quant_weight_block(w_gu.cuda())
    d_g = w8.w8_quant_weight_block(w_d.cuda())
    gu_o = orc.quant_weight_block(bits(w_gu))
    d_o = orc.quant_weight_block(bits(w_d))
    return H, I, g, gu_g, d_g, gu_o, d_o


@pytest.mark.parametrize("M", [1, 8, 32, 256, 1024])
def test_mlp_chain_block_fp8(orc, mlp_block, M):
    """The MLP block in Block-FP8: rms_norm + 1x128-group quant -> gate_up GEMM (128 x 128
    weight blocks) -> silu_and_mul + group quant -> down GEMM, AUTO with PDL.  Producer
    codes and group scales bit for bit on whole sampled rows, the GEMMs within the GEMM
    bound against the oracle fed with the oracle's own codes."""
    H, I, g, gu_g, d_g, gu_o, d_o = mlp_block
    fmt = w8.W8_FMT_BLOCK_FP8
    x = synth.activations(M, H, seed=synth.SEED_BASE + 6 + 10 * M)
    xd, gd = x.cuda(), g.cuda()
    q1, s1 = w8.w8_rmsnorm_quant_group(xd, gd, 1e-6)
    gu = w8.w8_gemm(fmt, q1, s1, gu_g[0], gu_g[1], variant=AUTO_PDL)
    q2, s2 = w8.w8_silu_mul_quant_group(gu)
    y = w8.w8_gemm(fmt, q2, s2, d_g[0], d_g[1], variant=AUTO_PDL)
    torch.cuda.synchronize()
    assert np.array_equal(u8(gu_g[0]), gu_o[0]) and np.array_equal(gu_g[1].cpu().numpy(), gu_o[1])
    rows = list(range(M)) if M <= 8 else sorted(set(np.random.default_rng(M + 1).integers(0, M, 5).tolist()) | {0, M - 1})
    xr = x[rows].contiguous()
    oq1, os1 = orc.rmsnorm_quant_group(bits(xr), bits(g), 1e-6)
    assert np.array_equal(u8(q1)[rows], oq1) and np.array_equal(s1.cpu().numpy()[rows], os1)
    gu_bits, gu_ref, _ = orc.gemm(2, oq1, os1, gu_o[0], gu_o[1])
    gu_out = gu.float().cpu().double().numpy()[rows]
    assert np.max(np.abs(gu_out - gu_ref)) <= TOL_REL * np.max(np.abs(gu_ref)) + TOL_ABS
    oq2, os2 = orc.silu_mul_quant_group(gu_bits)
    _, y_ref, _ = orc.gemm(2, oq2, os2, d_o[0], d_o[1])
    yo = y.float().cpu().double().numpy()[rows]
    # as in the FP8 chain: a last-bit difference of the intermediate bf16 can move a code
    assert np.max(np.abs(yo - y_ref)) <= TOL_REL * np.max(np.abs(y_ref)) + TOL_ABS
    assert w8.w8_device_status(clear=True) == 0
