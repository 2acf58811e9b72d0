"""Shared helpers for the GPU parity tests (inputs from the seeded generators; expected
values only from the CPU oracle)."""
import numpy as np
import torch

from bit_quantized_gemm_token_b200 import synth

TOL_REL = 2.0 ** -7
TOL_ABS = 1e-3


def bits(t):
    return synth.bf16_bits(t.cpu())


def u8(t):
    """Raw bytes of a CUDA/CPU 8-bit tensor as numpy uint8."""
    return t.cpu().contiguous().view(torch.uint8).numpy()


def assert_bf16_close(out_dev, ref_f64, what=""):
    """max|out - ref| <= 2^-7 max|ref| + 1e-3 (the GEMM acceptance bound)."""
    out = out_dev.float().cpu().double().numpy()
    ref = np.asarray(ref_f64, dtype=np.float64)
    assert out.shape == ref.shape, (out.shape, ref.shape)
    if out.size == 0:
        return
    err = np.max(np.abs(out - ref))
    bound = TOL_REL * np.max(np.abs(ref)) + TOL_ABS
    assert np.all(np.isfinite(out)), what + " non-finite output"
    assert err <= bound, "%s max err %.3g > bound %.3g" % (what, err, bound)


def quantize_operands(orc, fmt, x, w, ue8m0=False):
    """Oracle-side quantization of activations x[M,K] and weights w[N,K] (bf16, CPU)."""
    if fmt == 1:
        Aq, sA = orc.quant_rows(1, bits(x))
        Wq, sW = orc.quant_rows(1, bits(w))
    elif fmt == 0:
        Aq, sA = orc.quant_rows(0, bits(x))
        Wq, sW = orc.quant_rows(0, bits(w))
    else:
        Aq, sA = orc.quant_rows(0, bits(x), group=128, ue8m0=ue8m0)
        Wq, sW = orc.quant_weight_block(bits(w), ue8m0=ue8m0)
    return Aq, sA, Wq, sW


def dev_codes(a, fmt):
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.uint8))
    return t.view(torch.int8 if fmt == 1 else torch.float8_e4m3fn).cuda()


def dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def poison_bf16(shape):
    """Output buffer pre-filled with a NaN pattern, so unwritten elements show up."""
    return torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
