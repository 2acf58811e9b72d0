"""The allocation-free GEMM entry point (w8_gemm_noalloc), for callers that may not
call cudaMalloc -- e.g. code inside a runtime whose allocator it does not own, or a
service whose device memory is fixed at start-up.  Through the C ABI it must give
exactly what w8_gemm gives with a caller-provided workspace and the same variant (the
partial sums are added in a fixed order, so the two are bit-identical), on repeated
calls (its scratch array keeps the previous call's contents), stay within the GEMM
tolerance of the CPU oracle, leave the device's free memory unchanged once the first
call has been made, and reject variants whose scratch would exceed the array.  This
file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from bit_quantized_gemm_token_b200 import synth, w8
from gpu_helpers import assert_bf16_close, quantize_operands

pytestmark = pytest.mark.gpu


def _lib():
    L = w8.lib()
    f = L.w8_gemm_noalloc
    f.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def _P(t):
    return ctypes.c_void_p(t.data_ptr())


def _operands(fmt, M, N, K):
    x = synth.activations(M, K, seed=77).cuda()
    w = synth.weights(N, K, seed=78).cuda()
    if fmt == w8.W8_FMT_BLOCK_FP8:
        A, sA = w8.w8_quant_per_token(x, w8.W8_Q_FP8, group=128)
        W, sW = w8.w8_quant_weight_block(w)
    else:
        qf = w8.W8_Q_INT8 if fmt == w8.W8_FMT_INT8 else w8.W8_Q_FP8
        A, sA = w8.w8_quant_per_token(x, qf)
        W, sW = w8.w8_quant_per_token(w, qf)
    return A, sA, W, sW


CASES = [(w8.W8_FMT_FP8_DYN, "split8"), (w8.W8_FMT_FP8_DYN, "stream"), (w8.W8_FMT_FP8_DYN, "auto"),
         (w8.W8_FMT_INT8, "split8"), (w8.W8_FMT_INT8, "stream"), (w8.W8_FMT_INT8, "auto"),
         (w8.W8_FMT_BLOCK_FP8, "split4"), (w8.W8_FMT_BLOCK_FP8, "stream")]


@pytest.mark.parametrize("fmt,vdesc", CASES)
def test_noalloc_matches_workspace_gemm(fmt, vdesc):
    f = _lib()
    torch.cuda.set_device(0)
    M, N, K = 16, 2048, 4096
    A, sA, W, sW = _operands(fmt, M, N, K)
    v = {"split8": w8.variant(True, 8, 16), "split4": w8.variant(True, 4, 16),
         "stream": w8.variant(True, 1, 16, stream=True), "auto": w8.W8_VARIANT_AUTO}[vdesc]
    ref = w8.w8_gemm(fmt, A, sA, W, sW, variant=v, workspace=w8.Workspace())
    outs = [torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    free = []
    for out in outs:   # the second call finds the first call's contents in the scratch array
        free.append(torch.cuda.mem_get_info()[0])
        rc = f(fmt, _P(A), _P(sA), _P(W), _P(sW), _P(out), M, N, K, v, s)
        assert rc == w8.W8_OK, w8.status_string(rc)
        torch.cuda.synchronize()
    free.append(torch.cuda.mem_get_info()[0])
    for i, out in enumerate(outs):
        assert torch.equal(out, ref), "call %d differs from w8_gemm with the same variant" % i
    # the first call may bring the array (and the kernels' code) onto the device under
    # lazy module loading; after it, a call takes no device memory at all
    assert free[2] == free[1], "device memory taken by a repeated call: %d bytes" % (free[1] - free[2])


def test_noalloc_against_oracle(orc):
    """One case checked against the CPU oracle directly (the codes are the oracle's)."""
    f = _lib()
    torch.cuda.set_device(0)
    M, N, K = 16, 2048, 4096
    x = synth.activations(M, K, seed=91)
    w = synth.weights(N, K, seed=92)
    Aq, sA, Wq, sW = quantize_operands(orc, 0, x, w)
    _, ref, _ = orc.gemm(0, Aq, sA, Wq, sW)
    dA = torch.from_numpy(np.ascontiguousarray(Aq).view(np.uint8)).view(torch.float8_e4m3fn).cuda()
    dW = torch.from_numpy(np.ascontiguousarray(Wq).view(np.uint8)).view(torch.float8_e4m3fn).cuda()
    dsA = torch.from_numpy(np.ascontiguousarray(sA, dtype=np.float32)).cuda()
    dsW = torch.from_numpy(np.ascontiguousarray(sW, dtype=np.float32)).cuda()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = f(0, _P(dA), _P(dsA), _P(dW), _P(dsW), _P(out), M, N, K, w8.variant(True, 8, 16), s)
        assert rc == w8.W8_OK, w8.status_string(rc)
        torch.cuda.synchronize()
        assert_bf16_close(out, ref, "w8_gemm_noalloc vs oracle")


def test_noalloc_rejects_scratch_beyond_maximum():
    f = _lib()
    M, N, K = 8, 24576, 32768
    v = w8.variant(True, 256, 16)                      # 192 tiles x 256 splits of partials
    assert w8.w8_gemm_workspace_size(0, M, N, K, v) > (8 << 20)
    A = torch.zeros((M, K), dtype=torch.float8_e4m3fn, device="cuda")
    W = torch.zeros((N, K), dtype=torch.float8_e4m3fn, device="cuda")
    sA = torch.ones(M, device="cuda")
    sW = torch.ones(N, device="cuda")
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert f(0, _P(A), _P(sA), _P(W), _P(sW), _P(out), M, N, K, v, s) == w8.W8_ERR_WORKSPACE
