"""The Python binding refuses tensors whose layout, element type or size differ from
what the C entry points assume (they take bare pointers, row-major), before any call;
on a machine without a GPU the remaining refusal is the device."""
import pytest
import torch

from bit_quantized_gemm_token_b200 import w8

b8 = torch.float8_e4m3fn


def codes(*shape):
    return torch.zeros(shape, dtype=b8)


def f32(*shape):
    return torch.ones(shape, dtype=torch.float32)


def test_gemm_layouts():
    M, N, K = 4, 256, 512
    A, W = codes(M, K), codes(N, K)
    # transposed view: same shape, not row-major
    At = codes(K, M).t()
    with pytest.raises(ValueError, match="contiguous"):
        w8.w8_gemm(0, At, f32(M), W, f32(N))
    with pytest.raises(TypeError, match="1-byte"):
        w8.w8_gemm(0, A.to(torch.float16), f32(M), W, f32(N))
    with pytest.raises(ValueError, match="elements"):
        w8.w8_gemm(0, A, f32(M + 1), W, f32(N))
    with pytest.raises(ValueError, match="elements"):       # Block-FP8 wants [M, K/128] / [N/128, K/128]
        w8.w8_gemm(2, A, f32(M), W, f32(N))
    with pytest.raises(TypeError, match="float32"):
        w8.w8_gemm(0, A, f32(M).double(), W, f32(N))
    with pytest.raises(ValueError, match="shape"):
        w8.w8_gemm(0, A, f32(M), W, f32(N), out=torch.empty((M, N + 1), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="expected"):
        w8.w8_gemm(0, A, f32(M), codes(N, K + 16), f32(N))
    # everything right but the device
    with pytest.raises(TypeError, match="CUDA"):
        w8.w8_gemm(0, A, f32(M), W, f32(N), out=torch.empty((M, N), dtype=torch.bfloat16))
    with pytest.raises(TypeError, match="CUDA"):
        w8.w8_gemm(2, A, f32(M, K // 128), W, f32(2, K // 128), out=torch.empty((M, N), dtype=torch.bfloat16))


def test_grouped_and_debug_layouts():
    T, E, N, K = 8, 3, 256, 512
    A, W = codes(T, K), codes(E, N, K)
    off = torch.zeros(E + 1, dtype=torch.int32)
    with pytest.raises(ValueError, match="expected"):
        w8.w8_grouped_gemm(0, A, f32(T), codes(E * N, K), f32(E, N), off)
    with pytest.raises(ValueError, match="contiguous"):
        w8.w8_grouped_gemm(0, codes(K, T).t(), f32(T), W, f32(E, N), off)
    with pytest.raises(ValueError, match="expected"):
        w8.w8_gemm_i32_debug(A, codes(N, K + 16))
    with pytest.raises(ValueError, match="shape"):
        w8.w8_gemm_i32_debug(A.view(torch.int8), codes(N, K).view(torch.int8),
                             acc=torch.empty((T, N + 1), dtype=torch.int32))
    with pytest.raises(ValueError, match="contiguous"):
        w8.w8_gemm_i32_debug(A.view(torch.int8), codes(N, K).view(torch.int8),
                             acc=torch.empty((N, T), dtype=torch.int32).t())


def test_quantizer_layouts():
    x = torch.zeros((4, 512), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="unit column stride"):
        w8.w8_quant_per_token(torch.zeros((512, 4), dtype=torch.bfloat16).t())
    with pytest.raises(ValueError, match="elements"):
        w8.w8_quant_per_token(x, q=codes(4, 511))
    with pytest.raises(ValueError, match="elements"):
        w8.w8_quant_per_token(x, group=128, scale=f32(4))
    with pytest.raises(ValueError, match="elements"):
        w8.w8_rmsnorm_quant(x, torch.ones(511, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="even"):
        w8.w8_silu_mul_quant(torch.zeros((4, 513), dtype=torch.bfloat16))
    # a strided x (row stride > K) is accepted up to the device check
    big = torch.zeros((4, 640), dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="CUDA"):
        w8.w8_quant_per_token(big[:, :512])
