"""The allocation-free GEMM entry point (w8_gemm_noalloc), for callers that may not
call cudaMalloc -- e.g. code inside a runtime whose allocator it does not own.  It
must give the same result as w8_gemm with a caller-provided workspace, on repeated
calls (its scratch array keeps the previous call's contents), and reject variants
whose scratch would exceed the array.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from bit_quantized_gemm_token_b200 import synth, w8
from gpu_helpers import TOL_ABS, TOL_REL

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


@pytest.mark.parametrize("fmt", [w8.W8_FMT_FP8_DYN, w8.W8_FMT_INT8])
@pytest.mark.parametrize("vdesc", ["split8", "stream", "auto"])
def test_noalloc_matches_workspace_gemm(fmt, vdesc):
    f = _lib()
    torch.cuda.set_device(0)
    M, N, K = 16, 2048, 4096
    qf = w8.W8_Q_INT8 if fmt == w8.W8_FMT_INT8 else w8.W8_Q_FP8
    A, sA = w8.w8_quant_per_token(synth.activations(M, K, seed=77).cuda(), qf)
    W, sW = w8.w8_quant_per_token(synth.weights(N, K, seed=78).cuda(), qf)
    v = {"split8": w8.variant(True, 8, 16), "stream": w8.variant(True, 1, 16, stream=True),
         "auto": w8.W8_VARIANT_AUTO}[vdesc]
    ref = w8.w8_gemm(fmt, A, sA, W, sW, variant=v, workspace=w8.Workspace())
    torch.cuda.synchronize()
    refd = ref.float().cpu().double().numpy()
    bound = TOL_REL * np.max(np.abs(refd)) + TOL_ABS
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):   # the second call finds the first call's contents in the scratch array
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = f(fmt, _P(A), _P(sA), _P(W), _P(sW), _P(out), M, N, K, v, s)
        assert rc == w8.W8_OK, w8.status_string(rc)
        torch.cuda.synchronize()
        got = out.float().cpu().double().numpy()
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - refd)) <= bound


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
