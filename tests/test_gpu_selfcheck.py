"""The quantizers' division-free quotient gives the codes of the IEEE quotient x / s
that defines them, and the same fp32 quotient wherever a code can depend on it: an
exhaustive device-side enumeration of all bf16 pairs (x, amax) with |x| <= amax (amax up
to +inf), both signs, and 2^30 hashed fp32 pairs concentrated near the codes' rounding
midpoints, under the three scale rules (e4m3 per token, int8 per token, UE8M0 groups),
through the C ABI.  (Markstein's correction: "Computation of elementary functions on the
IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990; the codes follow "PyTorch
integra Helion en vLLM para acelerar inferencia FP8", section "Kernels Helion
implementados".)"""
import ctypes

import pytest
import torch

from bit_quantized_gemm_token_b200 import w8

pytestmark = pytest.mark.gpu


def _fn():
    f = w8.lib().w8_selfcheck_quotient
    f.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


@pytest.mark.parametrize("mode", [0, 1, 2, 3, 4, 5])
def test_quotient_matches_division(mode):
    f = _fn()
    torch.cuda.set_device(0)
    count = torch.zeros(1, dtype=torch.int64, device="cuda")
    first = torch.zeros(2, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream()
    rc = f(mode, ctypes.c_void_p(count.data_ptr()), ctypes.c_void_p(first.data_ptr()), ctypes.c_void_p(s.cuda_stream))
    assert rc == w8.W8_OK, w8.status_string(rc)
    torch.cuda.synchronize()
    n = int(count.item())
    fa, fx = (int(v) & 0xFFFFFFFF for v in first.cpu())
    assert n == 0, "%d pairs differ, e.g. amax bits 0x%08x, x bits 0x%08x" % (n, fa & 0x7FFFFFFF, fx)


def test_selfcheck_rejects_bad_arguments():
    f = _fn()
    assert f(6, None, None, None) == w8.W8_ERR_INVALID_ARG
    assert f(-1, None, None, None) == w8.W8_ERR_INVALID_ARG
