"""numpy front end for the C oracle (w8_oracle.c), loaded with ctypes.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Every function here only
marshals numpy arrays in and out of the C oracle; the arithmetic lives in C.

Conventions: bf16 tensors travel as their raw 16-bit patterns (np.uint16); 8-bit codes
as np.uint8 (e4m3) or np.int8 (int8); scales as np.float32.
"""
import ctypes
import os

import numpy as np

from . import build_oracle

Q_FP8, Q_INT8 = 0, 1
FMT_FP8_DYN, FMT_INT8, FMT_BLOCK_FP8 = 0, 1, 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        # W8_ORACLE_LIB: another build of the same C source (the mutation test loads
        # copies with a planted mistake this way)
        path = os.environ.get("W8_ORACLE_LIB") or build_oracle.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i, f = ctypes.c_int, ctypes.c_float
        L.orc_bf16_to_float.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_float.restype = f
        L.orc_bf16_from_double.argtypes = [ctypes.c_double]
        L.orc_bf16_from_double.restype = ctypes.c_uint16
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_encode.argtypes = [f]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_int8_encode.argtypes = [f]
        L.orc_int8_encode.restype = ctypes.c_int8
        L.orc_scale.argtypes = [f, f, i]
        L.orc_scale.restype = f
        L.orc_exp_f32.argtypes = [f]
        L.orc_exp_f32.restype = f
        L.orc_quant_rows.argtypes = [i, P, i, i, i, P, P, i, i]
        L.orc_quant_rows.restype = i
        L.orc_quant_weight_block.argtypes = [P, i, i, P, P, i]
        L.orc_quant_weight_block.restype = i
        L.orc_sumsq_f32.argtypes = [P, i]
        L.orc_sumsq_f32.restype = f
        L.orc_rmsnorm_f32.argtypes = [P, P, f, i, i, i, P]
        L.orc_rmsnorm_f32.restype = None
        L.orc_rmsnorm_quant.argtypes = [P, P, f, i, i, i, P, P]
        L.orc_rmsnorm_quant.restype = i
        L.orc_silu_mul_f32.argtypes = [P, i, i, i, P]
        L.orc_silu_mul_f32.restype = None
        L.orc_silu_mul_quant.argtypes = [P, i, i, i, P, P]
        L.orc_silu_mul_quant.restype = i
        L.orc_rmsnorm_quant_group.argtypes = [P, P, f, i, i, i, i, i, P, P]
        L.orc_rmsnorm_quant_group.restype = i
        L.orc_silu_mul_quant_group.argtypes = [P, i, i, i, i, i, P, P]
        L.orc_silu_mul_quant_group.restype = i
        L.orc_gemm.argtypes = [i, P, P, P, P, i, i, i, i, i, P, P, P]
        L.orc_qk_norm_rope.argtypes = [P, P, i, i, i, i, P, P, P, i, P, f]
        L.orc_gemm.restype = None
        L.orc_gemm_points.argtypes = [i, P, P, P, P, i, i, i, i, P, P, P]
        L.orc_gemm_points.restype = None
        L.orc_gemm_swap_ab.argtypes = [i, P, P, P, P, i, i, i, P]
        L.orc_gemm_swap_ab.restype = None
        L.orc_gemm_split_k.argtypes = [i, P, P, P, P, i, i, i, i, P]
        L.orc_gemm_split_k.restype = i
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --- scalar formats -------------------------------------------------------------

def e4m3_encode(v):
    v = np.asarray(v, dtype=np.float32)
    L = lib()
    return np.array([L.orc_e4m3_encode(float(x)) for x in v.ravel()], dtype=np.uint8).reshape(v.shape)


def e4m3_decode(c):
    c = np.asarray(c, dtype=np.uint8)
    L = lib()
    return np.array([L.orc_e4m3_decode(int(x)) for x in c.ravel()], dtype=np.float64).reshape(c.shape)


def int8_encode(v):
    v = np.asarray(v, dtype=np.float32)
    L = lib()
    return np.array([L.orc_int8_encode(float(x)) for x in v.ravel()], dtype=np.int8).reshape(v.shape)


def bf16_from_double(v):
    v = np.asarray(v, dtype=np.float64)
    L = lib()
    return np.array([L.orc_bf16_from_double(float(x)) for x in v.ravel()], dtype=np.uint16).reshape(v.shape)


def bf16_to_float(b):
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def scale(amax, qmax, ue8m0=False):
    return np.float32(lib().orc_scale(float(amax), float(qmax), int(bool(ue8m0))))


def exp_f32(x):
    x = np.asarray(x, dtype=np.float32)
    L = lib()
    return np.array([L.orc_exp_f32(float(v)) for v in x.ravel()], dtype=np.float32).reshape(x.shape)


# --- quantizers and producers -----------------------------------------------------

def quant_rows(qfmt, x_bits, group=0, ue8m0=False):
    """Per-token (group=0) or per-group quantization of bf16 rows x_bits[M, K]."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    q = np.zeros((M, K), dtype=np.uint8)
    ng = 1 if group == 0 else K // group
    s = np.zeros((M, ng), dtype=np.float32)
    rc = lib().orc_quant_rows(qfmt, _p(x), M, K, K, _p(q), _p(s), group, int(bool(ue8m0)))
    if rc != 0:
        raise ValueError("orc_quant_rows failed: %d" % rc)
    if qfmt == Q_INT8:
        q = q.view(np.int8)
    return q, (s[:, 0].copy() if group == 0 else s)


def quant_weight_block(w_bits, ue8m0=False):
    w = _c(w_bits, np.uint16)
    N, K = w.shape
    q = np.zeros((N, K), dtype=np.uint8)
    s = np.zeros(((N + 127) // 128, (K + 127) // 128), dtype=np.float32)
    lib().orc_quant_weight_block(_p(w), N, K, _p(q), _p(s), int(bool(ue8m0)))
    return q, s


def sumsq_f32(x_bits):
    """fp32 rounding (to nearest, ties to even) of the exact sum of squares of a 1-D
    array of bf16 values (raw bits)."""
    x = _c(x_bits, np.uint16).reshape(-1)
    return np.float32(lib().orc_sumsq_f32(_p(x), int(x.size)))


def rmsnorm_f32(x_bits, gamma_bits, eps):
    x = _c(x_bits, np.uint16)
    g = _c(gamma_bits, np.uint16)
    M, H = x.shape
    y = np.zeros((M, H), dtype=np.float32)
    lib().orc_rmsnorm_f32(_p(x), _p(g), float(eps), M, H, H, _p(y))
    return y


def rmsnorm_quant(x_bits, gamma_bits, eps):
    x = _c(x_bits, np.uint16)
    g = _c(gamma_bits, np.uint16)
    M, H = x.shape
    q = np.zeros((M, H), dtype=np.uint8)
    s = np.zeros((M,), dtype=np.float32)
    lib().orc_rmsnorm_quant(_p(x), _p(g), float(eps), M, H, H, _p(q), _p(s))
    return q, s


def silu_mul_f32(xgu_bits):
    x = _c(xgu_bits, np.uint16)
    M, I2 = x.shape
    I = I2 // 2
    h = np.zeros((M, I), dtype=np.float32)
    lib().orc_silu_mul_f32(_p(x), M, I, I2, _p(h))
    return h


def silu_mul_quant(xgu_bits):
    x = _c(xgu_bits, np.uint16)
    M, I2 = x.shape
    I = I2 // 2
    q = np.zeros((M, I), dtype=np.uint8)
    s = np.zeros((M,), dtype=np.float32)
    lib().orc_silu_mul_quant(_p(x), M, I, I2, _p(q), _p(s))
    return q, s


def rmsnorm_quant_group(x_bits, gamma_bits, eps, group=128, ue8m0=False):
    x = _c(x_bits, np.uint16)
    g = _c(gamma_bits, np.uint16)
    M, H = x.shape
    q = np.zeros((M, H), dtype=np.uint8)
    s = np.zeros((M, H // group), dtype=np.float32)
    rc = lib().orc_rmsnorm_quant_group(_p(x), _p(g), float(eps), M, H, H, group, int(bool(ue8m0)), _p(q), _p(s))
    if rc != 0:
        raise ValueError("orc_rmsnorm_quant_group failed: %d" % rc)
    return q, s


def silu_mul_quant_group(xgu_bits, group=128, ue8m0=False):
    x = _c(xgu_bits, np.uint16)
    M, I2 = x.shape
    I = I2 // 2
    q = np.zeros((M, I), dtype=np.uint8)
    s = np.zeros((M, I // group), dtype=np.float32)
    rc = lib().orc_silu_mul_quant_group(_p(x), M, I, I2, group, int(bool(ue8m0)), _p(q), _p(s))
    if rc != 0:
        raise ValueError("orc_silu_mul_quant_group failed: %d" % rc)
    return q, s


# --- GEMM -----------------------------------------------------------------------

def _gemm_args(Aq, sA, Wq, sW):
    Aq = _c(np.asarray(Aq).view(np.uint8), np.uint8)
    Wq = _c(np.asarray(Wq).view(np.uint8), np.uint8)
    sA = _c(sA, np.float32)
    sW = _c(sW, np.float32)
    return Aq, sA, Wq, sW


def gemm(fmt, Aq, sA, Wq, sW, n_lo=0, n_hi=None):
    """Returns (out_bf16_bits[M, w], ref_f64[M, w], acc_i64[M, w] or None) for columns
    [n_lo, n_hi)."""
    Aq, sA, Wq, sW = _gemm_args(Aq, sA, Wq, sW)
    M, K = Aq.shape
    N = Wq.shape[0]
    if n_hi is None:
        n_hi = N
    w = n_hi - n_lo
    out = np.zeros((M, w), dtype=np.uint16)
    ref = np.zeros((M, w), dtype=np.float64)
    acc = np.zeros((M, w), dtype=np.int64) if fmt == FMT_INT8 else None
    lib().orc_gemm(fmt, _p(Aq), _p(sA), _p(Wq), _p(sW), M, N, K, n_lo, n_hi, _p(out), _p(ref), _p(acc))
    return out, ref, acc


def gemm_ref_matmul(fmt, Aq, sA, Wq, sW):
    """The fp64 reference of orc_gemm (ref_f64) for every output, with numpy's matmul as
    the summation step: the codes are decoded with the oracle's own decoder (int8, or
    orc_e4m3_decode through a 256-entry table), each sum of products is exact in fp64 at
    these sizes (products of 8-bit values span < 2^36 and at most 2^15 of them are added),
    so any summation order gives orc_gemm's value; the scales are applied in orc_gemm's
    order -- (acc * sA) * sW, or per K block (sA * sW) * part added in block order.  For
    checking full-size outputs, where the C loop would take minutes."""
    Aq, sA, Wq, sW = _gemm_args(Aq, sA, Wq, sW)
    M, K = Aq.shape
    if fmt == FMT_INT8:
        a = Aq.view(np.int8).astype(np.float64)
        w = Wq.view(np.int8).astype(np.float64)
    else:
        table = e4m3_decode(np.arange(256, dtype=np.uint8))
        a = table[Aq]
        w = table[Wq]
    if fmt != FMT_BLOCK_FP8:
        acc = a @ w.T
        return (acc * sA.astype(np.float64)[:, None]) * sW.astype(np.float64)[None, :]
    nbk = (K + 127) // 128
    N = Wq.shape[0]
    ref = np.zeros((M, N), dtype=np.float64)
    sW2 = sW.reshape(-1, nbk).astype(np.float64)
    sA2 = sA.reshape(M, nbk).astype(np.float64)
    for kb in range(nbk):
        part = a[:, kb * 128:(kb + 1) * 128] @ w[:, kb * 128:(kb + 1) * 128].T
        sc = sA2[:, kb][:, None] * sW2[np.arange(N) // 128, kb][None, :]
        ref += sc * part
    return ref


def gemm_points(fmt, Aq, sA, Wq, sW, pm, pn):
    Aq, sA, Wq, sW = _gemm_args(Aq, sA, Wq, sW)
    M, K = Aq.shape
    N = Wq.shape[0]
    pm = _c(pm, np.int32)
    pn = _c(pn, np.int32)
    ref = np.zeros((len(pm),), dtype=np.float64)
    lib().orc_gemm_points(fmt, _p(Aq), _p(sA), _p(Wq), _p(sW), M, N, K, len(pm), _p(pm), _p(pn), _p(ref))
    return ref


def gemm_swap_ab(fmt, Aq, sA, Wq, sW):
    Aq, sA, Wq, sW = _gemm_args(Aq, sA, Wq, sW)
    M, K = Aq.shape
    N = Wq.shape[0]
    ref = np.zeros((M, N), dtype=np.float64)
    lib().orc_gemm_swap_ab(fmt, _p(Aq), _p(sA), _p(Wq), _p(sW), M, N, K, _p(ref))
    return ref


def gemm_split_k(fmt, Aq, sA, Wq, sW, S):
    Aq, sA, Wq, sW = _gemm_args(Aq, sA, Wq, sW)
    M, K = Aq.shape
    N = Wq.shape[0]
    ref = np.zeros((M, N), dtype=np.float64)
    rc = lib().orc_gemm_split_k(fmt, _p(Aq), _p(sA), _p(Wq), _p(sW), M, N, K, S, _p(ref))
    if rc != 0:
        raise ValueError("orc_gemm_split_k: bad split %d" % S)
    return ref


def bf16_max_err_ok(out_bits, ref_f64):
    """The GEMM acceptance bound: max|out - ref| <= 2^-7 * max|ref| + 1e-3."""
    out = bf16_to_float(out_bits).astype(np.float64)
    err = np.max(np.abs(out - ref_f64)) if out.size else 0.0
    bound = 2.0 ** -7 * (np.max(np.abs(ref_f64)) if ref_f64.size else 0.0) + 1e-3
    return err <= bound, err, bound


def qk_norm_rope(qkv_bits, Hq, Hkv, D, q_weight_bits, k_weight_bits, cos_sin, positions, eps=1e-6):
    """Per-head rms_norm of the query / key heads of qkv_bits[T, (Hq + 2 Hkv) * D], then
    rotate-halves rotary embedding with the fp32 table cos_sin[max_pos, D]; bf16 bits out."""
    x = _c(qkv_bits, np.uint16)
    T = x.shape[0]
    out = np.zeros_like(x)
    cs = _c(cos_sin, np.float32)
    pos = _c(positions, np.int64)
    rc = lib().orc_qk_norm_rope(_p(x), _p(out), T, Hq, Hkv, D, _p(_c(q_weight_bits, np.uint16)),
                                _p(_c(k_weight_bits, np.uint16)), _p(cs), cs.shape[0], _p(pos), float(eps))
    if rc != 0:
        raise ValueError("orc_qk_norm_rope failed: %d" % rc)
    return out


def grouped_gemm(fmt, Aq, sA, Wq, sW, offsets):
    """Grouped (mixture-of-experts) scaled GEMM: the activations' rows are sorted by
    expert, rows [offsets[e], offsets[e+1]) belong to expert e, and each is multiplied
    by that expert's weights Wq[e] [N, K] with its per-channel scales sW[e] [N]
    (FP8-dynamic, fmt 0, or W8A8-INT8, fmt 1): the plain GEMM of this module, expert by
    expert.  Returns (out_bf16_bits[T, N], ref_f64[T, N], acc_i64 or None)."""
    Aq = np.asarray(Aq)
    off = np.asarray(offsets, dtype=np.int64)
    E, N, K = np.asarray(Wq).shape
    T = Aq.shape[0]
    if off.shape != (E + 1,) or off[0] != 0 or off[-1] > T or np.any(np.diff(off) < 0):
        raise ValueError("offsets must rise from 0 to at most T")
    out = np.zeros((T, N), dtype=np.uint16)
    ref = np.zeros((T, N), dtype=np.float64)
    acc = np.zeros((T, N), dtype=np.int64) if fmt == 1 else None
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        o, r, a = gemm(fmt, Aq[lo:hi], np.asarray(sA)[lo:hi], np.asarray(Wq)[e], np.asarray(sW)[e])
        out[lo:hi], ref[lo:hi] = o, r
        if acc is not None:
            acc[lo:hi] = a
    return out, ref, acc
