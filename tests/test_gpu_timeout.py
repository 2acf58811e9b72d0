"""The bounded device waits end a kernel whose operands never arrive: the decode-form GEMM
run with its producer issuing no loads and a 1 ms bound on every wait records
W8_ERR_DEVICE_TIMEOUT in the device status word, returns, and leaves the context usable
-- the same GEMM then runs normally and matches the CPU oracle.  Nothing faults, traps or
spins without a bound: no copy or tensor-core instruction is ever in flight."""
import ctypes

import numpy as np
import pytest
import torch

from bit_quantized_gemm_token_b200 import synth, w8
from gpu_helpers import assert_bf16_close, quantize_operands, dev_codes, dev_f32

pytestmark = pytest.mark.gpu


def _fn():
    f = w8.lib().w8_gemm_timeout_debug
    f.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


@pytest.mark.parametrize("bn,c", [(128, 4), (256, 1)])
def test_wait_that_cannot_end_times_out_and_the_context_survives(orc, bn, c):
    torch.cuda.set_device(0)
    M, N, K = 8, 2048, 4096
    x = synth.activations(M, K, seed=911)
    w = synth.weights(N, K, seed=912)
    Aq, sA, Wq, sW = quantize_operands(orc, 0, x, w)
    _, ref, _ = orc.gemm(0, Aq, sA, Wq, sW)
    A, SA, W, SW = dev_codes(Aq, 0), dev_f32(sA), dev_codes(Wq, 0), dev_f32(sW)
    v = w8.decode_variant(bn, c, pdl=True)
    assert w8.w8_device_status(clear=True) == 0
    out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert _fn()(0, P(A), P(SA), P(W), P(SW), P(out), M, N, K, v, 1000, s) == w8.W8_OK
    torch.cuda.synchronize()
    assert w8.w8_device_status(clear=True) == w8.W8_ERR_DEVICE_TIMEOUT
    assert torch.isnan(out.float()).all()        # nothing written
    # the context is fine: the same GEMM, loads issued, normal bound
    good = w8.w8_gemm(0, A, SA, W, SW, variant=v)
    torch.cuda.synchronize()
    assert w8.w8_device_status(clear=True) == 0
    assert_bf16_close(good, ref, "after the timeout")


def test_timeout_debug_rejects_other_forms():
    M, N, K = 8, 2048, 4096
    A = torch.zeros((M, K), dtype=torch.float8_e4m3fn, device="cuda")
    W = torch.zeros((N, K), dtype=torch.float8_e4m3fn, device="cuda")
    sA, sW = torch.ones(M, device="cuda"), torch.ones(N, device="cuda")
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert _fn()(0, P(A), P(sA), P(W), P(sW), P(out), M, N, K, w8.variant(True, 1, 16, stream=True), 1000, s) == \
        w8.W8_ERR_UNSUPPORTED
    assert _fn()(0, P(A), P(sA), P(W), P(sW), P(out), M, N, K, 0, 0, s) == w8.W8_ERR_INVALID_ARG
