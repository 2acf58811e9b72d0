"""Seeded synthetic inputs for the 8-bit quantized linear layer.

This module only draws random numbers; it holds none of the layer's arithmetic (no
quantization, no scales, no GEMM), so both the CUDA path and the CPU oracle may take
their inputs from it.  Every tensor is created on the CPU with its own
torch.Generator, so a (seed, shape) pair always gives the same bytes; callers copy to
the GPU themselves.

Distributions (the synthetic stand-ins for a dense decoder's activations and weights;
no model weights or datasets are used):
  * activations: N(0, 1) bf16, with 0.1% of the elements (uniformly random positions)
    multiplied by 20 -- the outliers that make per-token scales matter;
  * weights:     N(0, 0.02) bf16, row-major [N, K] (out-features x in-features);
  * rms_norm gamma: U(0.5, 1.5) bf16;
  * rotary tables: fp32 [max_pos, D] rows (cos of D/2 angles, then their sines), from
    uniformly random angles, or the usual rotary angles pos * base^(-2i/D) of a
    decoder with rotary base `base` (an input of the query/key norm + rotary op, which
    takes the table as given).
"""
import torch

SEED_BASE = 1234          # seed = SEED_BASE + workload index (+ a per-tensor offset)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def activations(M: int, K: int, seed: int, outliers: bool = True) -> torch.Tensor:
    g = _gen(seed)
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    n = M * K
    if outliers and n > 0:
        cnt = max(1, n // 1000)
        idx = torch.randint(0, n, (cnt,), generator=g)
        x.view(-1)[idx] *= 20.0
    return x.to(torch.bfloat16)


def weights(N: int, K: int, seed: int, std: float = 0.02) -> torch.Tensor:
    g = _gen(seed)
    # drawn in row blocks to bound the fp32 temporary for very large matrices
    out = torch.empty(N, K, dtype=torch.bfloat16)
    step = max(1, (1 << 24) // max(1, K))
    for r in range(0, N, step):
        rows = min(step, N - r)
        out[r:r + rows] = (torch.randn(rows, K, generator=g, dtype=torch.float32) * std).to(torch.bfloat16)
    return out


def gamma(H: int, seed: int) -> torch.Tensor:
    g = _gen(seed)
    return (torch.rand(H, generator=g, dtype=torch.float32) + 0.5).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor):
    """Raw 16-bit patterns of a CPU bf16 tensor as a numpy uint16 array."""
    return t.contiguous().view(torch.int16).numpy().view("uint16")


def positions(T: int, max_pos: int, seed: int) -> torch.Tensor:
    g = _gen(seed)
    return torch.randint(0, max_pos, (T,), generator=g, dtype=torch.int64)


def rope_table(max_pos: int, D: int, seed: int = None, base: float = 1e6) -> torch.Tensor:
    """fp32 [max_pos, D]: columns [0, D/2) hold cos(a), [D/2, D) sin(a) of the angles a
    (random when a seed is given, else pos * base^(-2i/D)), computed in fp64."""
    half = D // 2
    if seed is not None:
        a = torch.rand(max_pos, half, generator=_gen(seed), dtype=torch.float64) * (2 * torch.pi)
    else:
        inv = base ** (-torch.arange(0, half, dtype=torch.float64) * 2.0 / D)
        a = torch.arange(max_pos, dtype=torch.float64)[:, None] * inv[None, :]
    return torch.cat([torch.cos(a), torch.sin(a)], dim=1).to(torch.float32)
