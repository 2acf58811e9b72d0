"""Python binding of libw8 (include/w8.h): the same entry points, argument marshalling
only.  Every step of the layer runs in the library's CUDA kernels; there is no CPU or
PyTorch-op fallback, and using any entry point without the built library raises.

Tensors are torch CUDA tensors.  Outputs may be passed in (for graph capture) or are
allocated here with torch (allocation is plumbing, not compute).  Calls are enqueued
on torch's current stream unless `stream` is given.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libw8.so")
DEFAULT_TABLE = os.path.join(_HERE, "tuning", "b200_table.txt")

# status codes
W8_OK = 0
W8_ERR_INVALID_ARG = -1
W8_ERR_UNSUPPORTED = -2
W8_ERR_ALIGNMENT = -3
W8_ERR_WORKSPACE = -4
W8_ERR_CUDA = -5
W8_ERR_DEVICE_TIMEOUT = -6
W8_ERR_NO_DEVICE = -7
W8_ERR_IO = -8

W8_Q_FP8, W8_Q_INT8 = 0, 1
W8_FMT_FP8_DYN, W8_FMT_INT8, W8_FMT_BLOCK_FP8, W8_FMT_BLOCK_FP8_UE8M0 = 0, 1, 2, 3

W8_VARIANT_AUTO = 0
W8_V_EXPLICIT = 1 << 0
W8_V_SWAP_AB = 1 << 1
W8_V_STREAM = 1 << 2
W8_V_SPLIT_SHIFT = 4
W8_V_TILE_SHIFT = 8
W8_V_STAGES_SHIFT = 12
W8_V_PDL = 1 << 16
W8_V_CLUSTER = 1 << 17
W8_V_BM64 = 1 << 18
W8_V_PFIX = 1 << 19
W8_V_FUSED = 1 << 24
W8_V_PAIR = 1 << 25
W8_V_DECODE = 1 << 26
W8_V_L2_SHIFT = 27
W8_V_KPS_SHIFT = 20
W8_V_CPS_SHIFT = 22
TILE_BN = {16: 0, 32: 1, 64: 2, 128: 3, 256: 4}


def variant(swap: bool, split: int = 1, bn: int = 16, stream: bool = False, stages: int = 0, pdl: bool = False,
            kps: int = 0, cps: int = 0, cluster: bool = False, bm64: bool = False, pfix: bool = False,
            pair: bool = False) -> int:
    """Explicit variant word (the W8_VARIANT macro plus stages, PDL, K blocks per stage
    and CTAs per SM)."""
    lg = int(split).bit_length() - 1
    if split < 1 or (1 << lg) != split:
        raise ValueError("split must be a power of two")
    v = W8_V_EXPLICIT | (W8_V_SWAP_AB if swap else 0) | (W8_V_STREAM if stream else 0)
    v |= (lg & 0xF) << W8_V_SPLIT_SHIFT
    v |= (TILE_BN[bn] & 0xF) << W8_V_TILE_SHIFT
    v |= (stages & 0xF) << W8_V_STAGES_SHIFT
    v |= (kps & 0x3) << W8_V_KPS_SHIFT
    v |= (cps & 0x3) << W8_V_CPS_SHIFT
    if pdl:
        v |= W8_V_PDL
    if cluster:
        v |= W8_V_CLUSTER
    if bm64:
        v |= W8_V_BM64
    if pfix:
        v |= W8_V_PFIX
    if pair:
        v |= W8_V_PAIR
    return v


def decode_variant(bn: int = 256, c: int = 1, stages: int = 0, l2ahead: int = 4, pdl: bool = False) -> int:
    """Explicit W8_V_DECODE variant word: bn weight rows per tile (64..256, a multiple of
    16), c K chunks per tile run as one cluster (1..8), stages (0 = default), l2ahead K
    blocks of weights kept in flight into L2 ahead of the stages."""
    if bn % 16 or not 64 <= bn <= 256:
        raise ValueError("bn must be a multiple of 16 in [64, 256]")
    if not 1 <= c <= 8:
        raise ValueError("c must be in [1, 8]")
    if not 0 <= l2ahead <= 15 or not 0 <= stages <= 15:
        raise ValueError("l2ahead and stages must be in [0, 15]")
    v = W8_V_EXPLICIT | W8_V_DECODE | ((c - 1) << W8_V_SPLIT_SHIFT) | ((bn // 16 - 1) << W8_V_TILE_SHIFT)
    v |= (stages << W8_V_STAGES_SHIFT) | (l2ahead << W8_V_L2_SHIFT)
    if pdl:
        v |= W8_V_PDL
    return v


def describe(v: int) -> dict:
    if v & W8_V_DECODE:
        return {"decode": True, "bn": 16 * (((v >> W8_V_TILE_SHIFT) & 0xF) + 1),
                "c": ((v >> W8_V_SPLIT_SHIFT) & 0xF) + 1, "stages": (v >> W8_V_STAGES_SHIFT) & 0xF,
                "l2ahead": (v >> W8_V_L2_SHIFT) & 0xF, "pdl": bool(v & W8_V_PDL),
                "swap_ab": False, "stream": False, "cluster": False, "bm64": False, "pfix": False, "pair": False}
    inv = {b: k for k, b in TILE_BN.items()}
    return {"decode": False, "swap_ab": bool(v & W8_V_SWAP_AB), "stream": bool(v & W8_V_STREAM),
            "split_k": 1 << ((v >> W8_V_SPLIT_SHIFT) & 0xF), "bn": inv.get((v >> W8_V_TILE_SHIFT) & 0xF),
            "stages": (v >> W8_V_STAGES_SHIFT) & 0xF, "pdl": bool(v & W8_V_PDL),
            "kps": (v >> W8_V_KPS_SHIFT) & 0x3, "cps": (v >> W8_V_CPS_SHIFT) & 0x3,
            "cluster": bool(v & W8_V_CLUSTER), "bm64": bool(v & W8_V_BM64), "pfix": bool(v & W8_V_PFIX),
            "pair": bool(v & W8_V_PAIR)}


class W8Error(RuntimeError):
    def __init__(self, fn, code):
        super().__init__("%s failed: %s (%d)" % (fn, status_string(code), code))
        self.code = code


_lib = None


def lib():
    """Load libw8.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libw8.so is not built: run `python -m bit_quantized_gemm_token_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.w8_quant_per_token.argtypes = [I, P, I, I, I, P, P, I, I, P]
    L.w8_quant_weight_block.argtypes = [P, I, I, P, P, I, P]
    L.w8_rmsnorm_quant.argtypes = [P, P, F, I, I, I, P, P, P]
    L.w8_silu_mul_quant.argtypes = [P, I, I, I, P, P, P]
    L.w8_rmsnorm_quant_group.argtypes = [P, P, F, I, I, I, I, I, P, P, P]
    L.w8_silu_mul_quant_group.argtypes = [P, I, I, I, I, I, P, P, P]
    L.w8_gemm.argtypes = [I, P, P, P, P, P, I, I, I, I, P, S, P]
    L.w8_gemm_workspace_size.argtypes = [I, I, I, I, I]
    L.w8_gemm_workspace_size.restype = S
    L.w8_gemm_resolve_variant.argtypes = [I, I, I, I, I]
    L.w8_gemm_i32_debug.argtypes = [P, P, P, I, I, I, I, P, S, P]
    L.w8_load_table.argtypes = [ctypes.c_char_p]
    L.w8_clear_table.argtypes = []
    L.w8_clear_table.restype = None
    L.w8_device_status.argtypes = [I]
    L.w8_status_string.argtypes = [I]
    L.w8_status_string.restype = ctypes.c_char_p
    L.w8_version.argtypes = []
    L.w8_linear.argtypes = [I, P, I, P, P, P, I, I, I, I, P, S, P]
    L.w8_qk_norm_rope.argtypes = [P, P, I, I, I, I, P, P, P, I, P, F, P]
    L.w8_grouped_gemm.argtypes = [I, P, P, P, P, P, P, I, I, I, I, I, I, P, S, P]
    L.w8_grouped_gemm_workspace_size.argtypes = [I, I, I, I, I, I, I]
    L.w8_grouped_gemm_workspace_size.restype = S
    L.w8_linear_debug.argtypes = [I, P, I, P, P, P, I, I, I, I, P, S, P, P, P]
    L.w8_linear_workspace_size.argtypes = [I, I, I, I, I]
    L.w8_linear_workspace_size.restype = S
    L.w8_linear_resolve.argtypes = [I, I, I, I, I]
    L.w8_linear_resolve.restype = I
    L.w8_gemm_occupancy.argtypes = [I, I, I, I, I]
    L.w8_gemm_occupancy.restype = I
    for fn in ("w8_linear", "w8_linear_debug", "w8_qk_norm_rope", "w8_grouped_gemm",
               "w8_quant_per_token", "w8_quant_weight_block", "w8_rmsnorm_quant", "w8_silu_mul_quant",
               "w8_rmsnorm_quant_group", "w8_silu_mul_quant_group", "w8_gemm",
               "w8_gemm_resolve_variant", "w8_gemm_i32_debug", "w8_load_table", "w8_device_status", "w8_version"):
        getattr(L, fn).restype = I
    _lib = L
    # the per-shape variant table shipped with the package (the offline sweep's output)
    # is loaded once; W8_TABLE=<path> picks another one, W8_TABLE=none loads none
    table = os.environ.get("W8_TABLE", DEFAULT_TABLE)
    if table != "none" and os.path.exists(table):
        n = L.w8_load_table(os.fsencode(table))
        if n < 0:
            raise W8Error("w8_load_table(%s)" % table, n)
    return L


def status_string(code: int) -> str:
    return lib().w8_status_string(int(code)).decode()


def _check(fn, rc):
    if rc != W8_OK:
        raise W8Error(fn, rc)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, name):
    if t.dtype != dtype or not t.is_cuda:
        raise TypeError("%s must be a CUDA %s tensor (got %s on %s)" % (name, dtype, t.dtype, t.device))


def _dense(t, name, dtype=None, numel=None, shape=None, codes=False):
    """t must be contiguous (row-major): the C entry points take bare pointers and
    assume that layout.  codes: any 1-byte element type (e4m3, int8 or raw
    bytes)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a tensor" % name)
    if codes and t.element_size() != 1:
        raise TypeError("%s must hold 1-byte codes (got %s)" % (name, t.dtype))
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s (got %s)" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous (row-major)" % name)
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s (got %s)" % (name, tuple(shape), tuple(t.shape)))
    if numel is not None and t.numel() != numel:
        raise ValueError("%s must have %d elements (got %d)" % (name, numel, t.numel()))


def _rows(t, name, dtype):
    """2-D tensor with unit column stride (its row stride is passed along)."""
    if not isinstance(t, torch.Tensor) or t.dtype != dtype:
        raise TypeError("%s must be a %s tensor" % (name, dtype))
    if t.dim() != 2 or t.stride(1) != 1 or t.stride(0) < t.shape[1]:
        raise ValueError("%s must be 2-D with unit column stride" % name)


def _cuda(**tensors):
    """After the layout checks: every tensor argument lives on the GPU."""
    for name, t in tensors.items():
        if not t.is_cuda:
            raise TypeError("%s must be a CUDA tensor (got %s)" % (name, t.device))


def _scale_counts(fmt, M, N, K):
    """Elements of the activation and weight scale arrays of a GEMM in format fmt."""
    if fmt >= W8_FMT_BLOCK_FP8:
        return M * (K // 128), ((N + 127) // 128) * (K // 128)
    return M, N


# ---------------------------------------------------------------------------- quantizers

def w8_quant_per_token(x, qfmt=W8_Q_FP8, group=0, ue8m0=False, q=None, scale=None, stream=None):
    """bf16 x[M, K] (row stride x.stride(0)) -> (codes[M, K], scales [M] or [M, K/group])."""
    _rows(x, "x", torch.bfloat16)
    M, K = x.shape
    qdt = torch.float8_e4m3fn if qfmt == W8_Q_FP8 else torch.int8
    if q is None:
        q = torch.empty((M, K), dtype=qdt, device=x.device)
    if scale is None:
        scale = torch.empty((M,) if group == 0 else (M, K // group), dtype=torch.float32, device=x.device)
    _dense(q, "q", numel=M * K, codes=True)
    _dense(scale, "scale", torch.float32, numel=M if group == 0 else M * (K // group))
    _cuda(x=x, q=q, scale=scale)
    rc = lib().w8_quant_per_token(qfmt, _ptr(x), M, K, x.stride(0), _ptr(q), _ptr(scale), group, int(bool(ue8m0)),
                                  _stream(stream))
    _check("w8_quant_per_token", rc)
    return q, scale


def w8_quant_weight_block(w, ue8m0=False, q=None, scale=None, stream=None):
    """bf16 W[N, K] -> (e4m3 codes [N, K], scales [ceil(N/128), ceil(K/128)])."""
    _need(w, torch.bfloat16, "w")
    N, K = w.shape
    if q is None:
        q = torch.empty((N, K), dtype=torch.float8_e4m3fn, device=w.device)
    if scale is None:
        scale = torch.empty(((N + 127) // 128, (K + 127) // 128), dtype=torch.float32, device=w.device)
    _dense(q, "q", numel=N * K, codes=True)
    _dense(scale, "scale", torch.float32, numel=((N + 127) // 128) * ((K + 127) // 128))
    _cuda(w=w, q=q, scale=scale)
    rc = lib().w8_quant_weight_block(_ptr(w.contiguous()), N, K, _ptr(q), _ptr(scale), int(bool(ue8m0)),
                                     _stream(stream))
    _check("w8_quant_weight_block", rc)
    return q, scale


def w8_rmsnorm_quant(x, gamma, eps=1e-6, q=None, scale=None, stream=None):
    _rows(x, "x", torch.bfloat16)
    M, H = x.shape
    _dense(gamma, "gamma", torch.bfloat16, numel=H)
    if q is None:
        q = torch.empty((M, H), dtype=torch.float8_e4m3fn, device=x.device)
    if scale is None:
        scale = torch.empty((M,), dtype=torch.float32, device=x.device)
    _dense(q, "q", numel=M * H, codes=True)
    _dense(scale, "scale", torch.float32, numel=M)
    _cuda(x=x, gamma=gamma, q=q, scale=scale)
    rc = lib().w8_rmsnorm_quant(_ptr(x), _ptr(gamma), float(eps), M, H, x.stride(0), _ptr(q), _ptr(scale),
                                _stream(stream))
    _check("w8_rmsnorm_quant", rc)
    return q, scale


def w8_silu_mul_quant(gate_up, q=None, scale=None, stream=None):
    """bf16 gate_up[M, 2I] (gate first) -> (e4m3 codes of silu(gate)*up [M, I], scales [M])."""
    _rows(gate_up, "gate_up", torch.bfloat16)
    M, I2 = gate_up.shape
    if I2 % 2:
        raise ValueError("gate_up must have an even number of columns [gate | up]")
    I = I2 // 2
    if q is None:
        q = torch.empty((M, I), dtype=torch.float8_e4m3fn, device=gate_up.device)
    if scale is None:
        scale = torch.empty((M,), dtype=torch.float32, device=gate_up.device)
    _dense(q, "q", numel=M * I, codes=True)
    _dense(scale, "scale", torch.float32, numel=M)
    _cuda(gate_up=gate_up, q=q, scale=scale)
    rc = lib().w8_silu_mul_quant(_ptr(gate_up), M, I, gate_up.stride(0), _ptr(q), _ptr(scale), _stream(stream))
    _check("w8_silu_mul_quant", rc)
    return q, scale


def w8_rmsnorm_quant_group(x, gamma, eps=1e-6, group=128, ue8m0=False, q=None, scale=None, stream=None):
    """rms_norm + 1x128-group fp8 quant: (e4m3 codes [M, H], scales [M, H/group])."""
    _rows(x, "x", torch.bfloat16)
    M, H = x.shape
    _dense(gamma, "gamma", torch.bfloat16, numel=H)
    if q is None:
        q = torch.empty((M, H), dtype=torch.float8_e4m3fn, device=x.device)
    if scale is None:
        scale = torch.empty((M, H // group), dtype=torch.float32, device=x.device)
    _dense(q, "q", numel=M * H, codes=True)
    _dense(scale, "scale", torch.float32, numel=M * (H // group))
    _cuda(x=x, gamma=gamma, q=q, scale=scale)
    rc = lib().w8_rmsnorm_quant_group(_ptr(x), _ptr(gamma), float(eps), M, H, x.stride(0), group, int(bool(ue8m0)),
                                      _ptr(q), _ptr(scale), _stream(stream))
    _check("w8_rmsnorm_quant_group", rc)
    return q, scale


def w8_silu_mul_quant_group(gate_up, group=128, ue8m0=False, q=None, scale=None, stream=None):
    """silu_and_mul + 1x128-group fp8 quant: (e4m3 codes [M, I], scales [M, I/group])."""
    _rows(gate_up, "gate_up", torch.bfloat16)
    M, I2 = gate_up.shape
    if I2 % 2:
        raise ValueError("gate_up must have an even number of columns [gate | up]")
    I = I2 // 2
    if q is None:
        q = torch.empty((M, I), dtype=torch.float8_e4m3fn, device=gate_up.device)
    if scale is None:
        scale = torch.empty((M, I // group), dtype=torch.float32, device=gate_up.device)
    _dense(q, "q", numel=M * I, codes=True)
    _dense(scale, "scale", torch.float32, numel=M * (I // group))
    _cuda(gate_up=gate_up, q=q, scale=scale)
    rc = lib().w8_silu_mul_quant_group(_ptr(gate_up), M, I, gate_up.stride(0), group, int(bool(ue8m0)), _ptr(q),
                                       _ptr(scale), _stream(stream))
    _check("w8_silu_mul_quant_group", rc)
    return q, scale


# ---------------------------------------------------------------------------- GEMM

def w8_gemm_workspace_size(fmt, M, N, K, variant=W8_VARIANT_AUTO):
    n = lib().w8_gemm_workspace_size(fmt, M, N, K, variant)
    if n == ctypes.c_size_t(-1).value:
        raise W8Error("w8_gemm_workspace_size", W8_ERR_INVALID_ARG)
    return n


def w8_gemm_occupancy(fmt, M, N, K, variant=W8_VARIANT_AUTO):
    """CTAs of the selected GEMM kernel that fit on one SM together."""
    n = lib().w8_gemm_occupancy(fmt, M, N, K, variant)
    if n < 0:
        raise W8Error("w8_gemm_occupancy", n)
    return n


def w8_gemm_resolve_variant(fmt, M, N, K, variant=W8_VARIANT_AUTO):
    v = lib().w8_gemm_resolve_variant(fmt, M, N, K, variant)
    if v < 0:
        raise W8Error("w8_gemm_resolve_variant", v)
    return v


class Workspace:
    """A zero-initialised device scratch buffer for w8_gemm, grown on demand (growth
    re-zeroes).  Calls sharing one workspace must be ordered on one stream."""

    def __init__(self, device=None, nbytes=0):
        self.device = torch.device(device or "cuda")
        self.buf = None
        if nbytes:
            self.reserve(nbytes)

    def reserve(self, nbytes):
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.buf

    def args(self, nbytes):
        if nbytes == 0:
            return None, 0
        b = self.reserve(nbytes)
        return ctypes.c_void_p(b.data_ptr()), b.numel()


_default_ws = {}


def _workspace(ws, device, nbytes):
    if ws is None:
        ws = _default_ws.setdefault(device, Workspace(device))
    return ws.args(nbytes)


def w8_gemm(fmt, A_q, A_scale, W_q, W_scale, out=None, variant=W8_VARIANT_AUTO, workspace=None, stream=None):
    """out[M, N] (bf16) = scaled A_q . W_q^T in format `fmt` (W8_FMT_*)."""
    _dense(A_q, "A_q", codes=True)
    _dense(W_q, "W_q", codes=True)
    if A_q.dim() != 2 or W_q.dim() != 2 or W_q.shape[1] != A_q.shape[1]:
        raise ValueError("A_q [M, K] and W_q [N, K] expected")
    M, K = A_q.shape
    N = W_q.shape[0]
    na, nw = _scale_counts(fmt, M, N, K)
    _dense(A_scale, "A_scale", torch.float32, numel=na)
    _dense(W_scale, "W_scale", torch.float32, numel=nw)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A_q.device)
    _dense(out, "out", torch.bfloat16, shape=(M, N))
    _cuda(A_q=A_q, A_scale=A_scale, W_q=W_q, W_scale=W_scale, out=out)
    nbytes = w8_gemm_workspace_size(fmt, M, N, K, variant)
    wp, wn = _workspace(workspace, A_q.device, nbytes)
    rc = lib().w8_gemm(fmt, _ptr(A_q), _ptr(A_scale), _ptr(W_q), _ptr(W_scale), _ptr(out), M, N, K, variant, wp, wn,
                       _stream(stream))
    _check("w8_gemm", rc)
    return out


def w8_grouped_gemm_workspace_size(fmt, E, T, N, K, max_tokens_per_expert, variant=W8_VARIANT_AUTO):
    n = lib().w8_grouped_gemm_workspace_size(fmt, E, T, N, K, max_tokens_per_expert, variant)
    if n == ctypes.c_size_t(-1).value:
        raise W8Error("w8_grouped_gemm_workspace_size", W8_ERR_INVALID_ARG)
    return n


def w8_grouped_gemm(fmt, A_q, A_scale, W_q, W_scale, expert_offsets, max_tokens_per_expert=None, out=None,
                    variant=W8_VARIANT_AUTO, workspace=None, stream=None):
    """Mixture-of-experts GEMM: A_q [T, K] rows sorted by expert (rows [off[e], off[e+1])
    belong to expert e), W_q [E, N, K], W_scale [E, N]; expert_offsets int32 [E+1] on the
    device.  Rows no expert owns are left as they were in `out`."""
    _dense(A_q, "A_q", codes=True)
    _dense(W_q, "W_q", codes=True)
    if A_q.dim() != 2 or W_q.dim() != 3 or W_q.shape[2] != A_q.shape[1]:
        raise ValueError("A_q [T, K] and W_q [E, N, K] expected")
    T, K = A_q.shape
    E, N, _ = W_q.shape
    if expert_offsets.dtype != torch.int32 or not expert_offsets.is_cuda or expert_offsets.numel() != E + 1:
        raise TypeError("expert_offsets must be a CUDA int32 tensor of E + 1 entries")
    _dense(expert_offsets, "expert_offsets", torch.int32)
    _dense(A_scale, "A_scale", torch.float32, numel=T)
    _dense(W_scale, "W_scale", torch.float32, numel=E * N)
    mm = T if max_tokens_per_expert is None else int(max_tokens_per_expert)
    if out is None:
        out = torch.zeros((T, N), dtype=torch.bfloat16, device=A_q.device)
    _dense(out, "out", torch.bfloat16, shape=(T, N))
    _cuda(A_q=A_q, A_scale=A_scale, W_q=W_q, W_scale=W_scale, out=out, expert_offsets=expert_offsets)
    nbytes = w8_grouped_gemm_workspace_size(fmt, E, T, N, K, mm, variant)
    wp, wn = _workspace(workspace, A_q.device, nbytes)
    rc = lib().w8_grouped_gemm(fmt, _ptr(A_q), _ptr(A_scale), _ptr(W_q), _ptr(W_scale), _ptr(out),
                               _ptr(expert_offsets), E, T, N, K, mm, variant, wp, wn, _stream(stream))
    _check("w8_grouped_gemm", rc)
    return out


def w8_qk_norm_rope(qkv, Hq, Hkv, D, q_weight, k_weight, cos_sin, positions, eps=1e-6, out=None, stream=None):
    """Query/key per-head rms_norm + rotary embedding of qkv [T, (Hq + 2 Hkv) * D] bf16;
    out=qkv works in place.  cos_sin fp32 [max_pos, D]; positions int64 [T]."""
    _need(qkv, torch.bfloat16, "qkv")
    T = qkv.shape[0]
    if qkv.shape[1] != (Hq + 2 * Hkv) * D or not qkv.is_contiguous():
        raise ValueError("qkv must be contiguous [T, (Hq + 2 Hkv) * D]")
    if out is None:
        out = torch.empty_like(qkv)
    _dense(out, "out", torch.bfloat16, shape=tuple(qkv.shape))
    _dense(q_weight, "q_weight", torch.bfloat16, numel=D)
    _dense(k_weight, "k_weight", torch.bfloat16, numel=D)
    _dense(cos_sin, "cos_sin", torch.float32)
    if cos_sin.dim() != 2 or cos_sin.shape[1] != D:
        raise ValueError("cos_sin must be [max_pos, D]")
    _dense(positions, "positions", torch.int64, numel=T)
    _cuda(qkv=qkv, out=out, q_weight=q_weight, k_weight=k_weight, cos_sin=cos_sin, positions=positions)
    rc = lib().w8_qk_norm_rope(_ptr(qkv), _ptr(out), T, Hq, Hkv, D, _ptr(q_weight), _ptr(k_weight), _ptr(cos_sin),
                               cos_sin.shape[0], _ptr(positions), float(eps), _stream(stream))
    _check("w8_qk_norm_rope", rc)
    return out


def w8_linear_workspace_size(fmt, M, N, K, variant=W8_VARIANT_AUTO):
    n = lib().w8_linear_workspace_size(fmt, M, N, K, variant)
    if n == ctypes.c_size_t(-1).value:
        raise W8Error("w8_linear_workspace_size", W8_ERR_INVALID_ARG)
    return n


def w8_linear_resolve(fmt, M, N, K, variant=W8_VARIANT_AUTO):
    """The explicit variant w8_linear runs (W8_V_FUSED set for the one-kernel form)."""
    v = lib().w8_linear_resolve(fmt, M, N, K, variant)
    if v < 0:
        raise W8Error("w8_linear_resolve", v)
    return v


def w8_linear(fmt, x, W_q, W_scale, out=None, variant=W8_VARIANT_AUTO, workspace=None, stream=None):
    """out[M, N] (bf16) = scaled quant(x) . W_q^T: x bf16 [M, K] quantized per token (or
    per 1 x 128 group for Block-FP8) and multiplied in one call: the quantizer and the
    GEMM, or one kernel when the variant carries W8_V_FUSED."""
    _rows(x, "x", torch.bfloat16)
    M, K = x.shape
    _dense(W_q, "W_q", codes=True)
    if W_q.dim() != 2 or W_q.shape[1] != K:
        raise ValueError("W_q [N, K] expected")
    N = W_q.shape[0]
    _dense(W_scale, "W_scale", torch.float32, numel=_scale_counts(fmt, M, N, K)[1])
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _dense(out, "out", torch.bfloat16, shape=(M, N))
    _cuda(x=x, W_q=W_q, W_scale=W_scale, out=out)
    nbytes = w8_linear_workspace_size(fmt, M, N, K, variant)
    wp, wn = _workspace(workspace, x.device, nbytes)
    rc = lib().w8_linear(fmt, _ptr(x), x.stride(0), _ptr(W_q), _ptr(W_scale), _ptr(out), M, N, K, variant, wp, wn,
                         _stream(stream))
    _check("w8_linear", rc)
    return out


def w8_linear_debug(fmt, x, W_q, W_scale, variant=W8_VARIANT_AUTO, workspace=None, stream=None):
    """One-kernel w8_linear that also returns the codes [M, K] (uint8) and scales it computed."""
    _rows(x, "x", torch.bfloat16)
    M, K = x.shape
    _dense(W_q, "W_q", codes=True)
    if W_q.dim() != 2 or W_q.shape[1] != K:
        raise ValueError("W_q [N, K] expected")
    N = W_q.shape[0]
    _dense(W_scale, "W_scale", torch.float32, numel=_scale_counts(fmt, M, N, K)[1])
    out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    q = torch.zeros((M, K), dtype=torch.uint8, device=x.device)
    s = torch.zeros((M, K // 128) if fmt >= W8_FMT_BLOCK_FP8 else (M,), dtype=torch.float32, device=x.device)
    _cuda(x=x, W_q=W_q, W_scale=W_scale)
    nbytes = w8_linear_workspace_size(fmt, M, N, K, variant)
    wp, wn = _workspace(workspace, x.device, nbytes)
    rc = lib().w8_linear_debug(fmt, _ptr(x), x.stride(0), _ptr(W_q), _ptr(W_scale), _ptr(out), M, N, K, variant, wp,
                               wn, _ptr(q), _ptr(s), _stream(stream))
    _check("w8_linear_debug", rc)
    return out, q, s


def w8_gemm_i32_debug(A_q, W_q, acc=None, variant=W8_VARIANT_AUTO, workspace=None, stream=None):
    """Raw int32 accumulators acc[M, N] = sum_k A_q W_q (INT8 path, no scales)."""
    _dense(A_q, "A_q", codes=True)
    _dense(W_q, "W_q", codes=True)
    if A_q.dim() != 2 or W_q.dim() != 2 or W_q.shape[1] != A_q.shape[1]:
        raise ValueError("A_q [M, K] and W_q [N, K] expected")
    M, K = A_q.shape
    N = W_q.shape[0]
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=A_q.device)
    _dense(acc, "acc", torch.int32, shape=(M, N))
    _cuda(A_q=A_q, W_q=W_q, acc=acc)
    nbytes = w8_gemm_workspace_size(W8_FMT_INT8, M, N, K, variant)
    wp, wn = _workspace(workspace, A_q.device, nbytes)
    rc = lib().w8_gemm_i32_debug(_ptr(A_q), _ptr(W_q), _ptr(acc), M, N, K, variant, wp, wn, _stream(stream))
    _check("w8_gemm_i32_debug", rc)
    return acc


def w8_load_table(path):
    n = lib().w8_load_table(os.fsencode(path))
    if n < 0:
        raise W8Error("w8_load_table", n)
    return n


def w8_clear_table():
    lib().w8_clear_table()


def w8_device_status(clear=True):
    return lib().w8_device_status(int(bool(clear)))


def w8_status_string(code):
    return status_string(code)


def w8_version():
    return lib().w8_version()
