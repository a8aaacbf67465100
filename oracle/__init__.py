"""CPU oracle for the W4A16 path -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference legs may
import this package.  The product path (bit_weight_only_w4_b200) never imports it and
shares no code with it.

Thin numpy wrappers around the plain C functions in w4_oracle.c; every function states
the passage it follows in the C source.  Arrays of 16-bit floats are passed as their
raw uint16 bit patterns so the oracle's own IEEE converters decide every rounding.

Parity of each function is pinned in tests/test_oracle_*.py (closed forms, brute force,
library routines, hand-worked fixtures under tests/golden/).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i64, i32, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
        L.oracle_f16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_f16_to_f32.restype = ctypes.c_float
        L.oracle_f32_to_f16.argtypes = [ctypes.c_float]
        L.oracle_f32_to_f16.restype = ctypes.c_uint16
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f32.restype = ctypes.c_float
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        for name in ("oracle_f16_to_f32_array", "oracle_f32_to_f16_array",
                     "oracle_bf16_to_f32_array", "oracle_f32_to_bf16_array"):
            getattr(L, name).argtypes = [vp, i64, vp]
            getattr(L, name).restype = None
        L.oracle_awq_scale_weights.argtypes = [vp, ctypes.c_int, i64, i64, vp, vp]
        L.oracle_awq_scale_acts.argtypes = [vp, ctypes.c_int, i64, i64, vp, vp]
        L.oracle_quantize.argtypes = [vp, i64, i64, i32, ctypes.c_int, vp, vp, vp, vp]
        L.oracle_quantize.restype = ctypes.c_int
        L.oracle_pack_canonical.argtypes = [vp, i64, i64, vp]
        L.oracle_unpack_canonical.argtypes = [vp, i64, i64, vp]
        L.oracle_pack_device.argtypes = [vp, i64, i64, vp]
        L.oracle_pack_device.restype = ctypes.c_int
        L.oracle_unpack_device.argtypes = [vp, i64, i64, vp]
        L.oracle_unpack_device.restype = ctypes.c_int
        L.oracle_dequant.argtypes = [vp, vp, vp, vp, i32, i64, i64, vp]
        L.oracle_gemm_f32.argtypes = [vp, vp, i64, i64, i64, vp, i64, vp]
        L.oracle_gemm_f64.argtypes = [vp, vp, i64, i64, i64, vp, i64, vp]
        L.oracle_e2m1_to_f32.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_to_f32.restype = ctypes.c_float
        L.oracle_f32_to_e2m1.argtypes = [ctypes.c_float]
        L.oracle_f32_to_e2m1.restype = ctypes.c_uint8
        L.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_to_f32.restype = ctypes.c_float
        L.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
        L.oracle_f32_to_e4m3.restype = ctypes.c_uint8
        L.oracle_nvfp4_quantize.argtypes = [vp, ctypes.c_int, i64, i64, vp, vp, vp]
        L.oracle_nvfp4_quantize.restype = ctypes.c_int
        L.oracle_nvfp4_dequant.argtypes = [vp, vp, ctypes.c_float, i64, i64, vp]
        L.oracle_mxfp4_quantize.argtypes = [vp, ctypes.c_int, i64, i64, vp, vp]
        L.oracle_mxfp4_quantize.restype = ctypes.c_int
        L.oracle_mxfp4_dequant.argtypes = [vp, vp, i64, i64, vp]
        _LIB = L
    return _LIB


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def bits16(a):
    """Raw uint16 bit patterns of an fp16 / bf16 array (numpy float16 or uint16 input)."""
    a = np.asarray(a)
    if a.dtype == np.float16:
        return np.ascontiguousarray(a).view(np.uint16)
    if a.dtype == np.uint16:
        return np.ascontiguousarray(a)
    raise TypeError(f"expected float16 or uint16 bit patterns, got {a.dtype}")


# ---- IEEE conversions (written from the binary16 / bfloat16 definitions) ----------------
def f16_to_f32(h):
    h = bits16(h)
    out = np.empty(h.shape, np.float32)
    lib().oracle_f16_to_f32_array(_p(h), h.size, _p(out))
    return out


def f32_to_f16(f):
    f = _c(f, np.float32)
    out = np.empty(f.shape, np.uint16)
    lib().oracle_f32_to_f16_array(_p(f), f.size, _p(out))
    return out


def bf16_to_f32(h):
    h = bits16(h)
    out = np.empty(h.shape, np.float32)
    lib().oracle_bf16_to_f32_array(_p(h), h.size, _p(out))
    return out


def f32_to_bf16(f):
    f = _c(f, np.float32)
    out = np.empty(f.shape, np.uint16)
    lib().oracle_f32_to_bf16_array(_p(f), f.size, _p(out))
    return out


# ---- AWQ equivalence transform (eq. 1) -------------------------------------------------
def awq_scale_weights(W_bits, s=None, is_bf16=False):
    """W'[n,k] = fp32(W[n,k]) * s[k] (fp32).  W_bits: uint16 [N,K]."""
    W_bits = bits16(W_bits)
    N, K = W_bits.shape
    s = _c(s, np.float32)
    Wp = np.empty((N, K), np.float32)
    lib().oracle_awq_scale_weights(_p(W_bits), int(is_bf16), N, K, _p(s), _p(Wp))
    return Wp


def awq_scale_acts(X_bits, s_inv=None, is_bf16=False):
    """X'[m,k] = fp32(X[m,k]) * s_inv[k] (fp32).  X_bits: uint16 [M,K]."""
    X_bits = bits16(X_bits)
    M, K = X_bits.shape
    s_inv = _c(s_inv, np.float32)
    Xp = np.empty((M, K), np.float32)
    lib().oracle_awq_scale_acts(_p(X_bits), int(is_bf16), M, K, _p(s_inv), _p(Xp))
    return Xp


# ---- group-wise RTN INT4 ---------------------------------------------------------------
def quantize(Wp, group_size, symmetric=False, g_idx=None):
    """Quantise fp32 W' [N,K]; returns (q uint8 [N,K], scales uint16 [G,N], zeros uint16 [G,N] or None)."""
    Wp = _c(Wp, np.float32)
    N, K = Wp.shape
    G = K // group_size
    g_idx = _c(g_idx, np.int32)
    q = np.empty((N, K), np.uint8)
    scales = np.empty((G, N), np.uint16)
    zeros = None if symmetric else np.empty((G, N), np.uint16)
    rc = lib().oracle_quantize(_p(Wp), N, K, int(group_size), int(bool(symmetric)), _p(g_idx),
                               _p(q), _p(scales), _p(zeros))
    if rc != 0:
        raise ValueError("oracle_quantize rejected its arguments")
    return q, scales, zeros


def quantize_weights(W_bits, s, group_size, symmetric=False, g_idx=None, is_bf16=False):
    """Steps in the pages' order: AWQ weight scaling, then group-wise RTN."""
    return quantize(awq_scale_weights(W_bits, s, is_bf16), group_size, symmetric, g_idx)


# ---- packing -------------------------------------------------------------------------
def pack_canonical(q):
    q = _c(q, np.uint8)
    N, K = q.shape
    out = np.empty((N, K // 8), np.uint32)
    lib().oracle_pack_canonical(_p(q), N, K, _p(out))
    return out


def unpack_canonical(qc, K):
    qc = _c(qc, np.uint32)
    N = qc.shape[0]
    out = np.empty((N, K), np.uint8)
    lib().oracle_unpack_canonical(_p(qc), N, K, _p(out))
    return out


def pack_device(q):
    q = _c(q, np.uint8)
    N, K = q.shape
    out = np.empty(N * K // 8, np.uint32)
    if lib().oracle_pack_device(_p(q), N, K, _p(out)) != 0:
        raise ValueError("device packing needs N % 16 == 0 and K % 64 == 0")
    return out


def unpack_device(qd, N, K):
    qd = _c(qd, np.uint32).reshape(-1)
    out = np.empty((N, K), np.uint8)
    if lib().oracle_unpack_device(_p(qd), N, K, _p(out)) != 0:
        raise ValueError("device packing needs N % 16 == 0 and K % 64 == 0")
    return out


# ---- dequantisation and the reference product ----------------------------------------
def dequant(q, scales, zeros, group_size, g_idx=None):
    q = _c(q, np.uint8)
    N, K = q.shape
    scales = bits16(scales)
    zeros = None if zeros is None else bits16(zeros)
    g_idx = _c(g_idx, np.int32)
    What = np.empty((N, K), np.float32)
    lib().oracle_dequant(_p(q), _p(scales), _p(zeros), _p(g_idx), int(group_size), N, K, _p(What))
    return What


def gemm_f32(Xp, What, rows=None):
    """Y[i,n] = sum_k X'[rows[i],k] What[n,k], fp32 accumulation in ascending k."""
    Xp = _c(Xp, np.float32)
    What = _c(What, np.float32)
    M, K = Xp.shape
    N = What.shape[0]
    rows = _c(rows, np.int64)
    R = M if rows is None else rows.size
    Y = np.empty((R, N), np.float32)
    lib().oracle_gemm_f32(_p(Xp), _p(What), M, N, K, _p(rows), 0 if rows is None else R, _p(Y))
    return Y


def gemm_f64(Xp, What, rows=None):
    Xp = _c(Xp, np.float32)
    What = _c(What, np.float32)
    M, K = Xp.shape
    N = What.shape[0]
    rows = _c(rows, np.int64)
    R = M if rows is None else rows.size
    Y = np.empty((R, N), np.float64)
    lib().oracle_gemm_f64(_p(Xp), _p(What), M, N, K, _p(rows), 0 if rows is None else R, _p(Y))
    return Y


def reference_y(X_bits, s_inv, q, scales, zeros, group_size, g_idx=None, x_is_bf16=False,
                rows=None):
    """The whole online path in the pages' order: X' = X s^-1, What = dequant, Y = X' What^T."""
    Xp = awq_scale_acts(X_bits, s_inv, x_is_bf16)
    What = dequant(q, scales, zeros, group_size, g_idx)
    return gemm_f32(Xp, What, rows)


# ---- AWQ scale search ----------------------------------------------------------------
def awq_search(W_bits, X_bits, group_size, symmetric=False, n_grid=20, w_is_bf16=False, x_is_bf16=False):
    """AWQ's per-channel scale search ("Quantization Paradigms for Edge Inference: AWQ, GPTQ,
    and FP8 Matrix Cores", sec. 3, eq. 2: s minimises || W X - Q(W diag(s)) diag(s)^-1 X ||_2,
    s found from activation magnitudes), over the candidates
        s_j = fp32(exp(a_j (log m - mean(log m)))),  m[k] = mean_i |X[i,k]|,  a_j = j / n_grid,
    in plain steps: m and its logarithms in fp64; per candidate the oracle's quantiser on
    W diag(s_j), X' = X s_j^-1 rounded to the activation type (as the GEMM does), the fp32
    product X' What^T, and the squared error against the fp32 product X W^T summed in fp64.
    Returns (first index of the smallest loss, losses fp64 [n_grid], s of that index)."""
    X_bits = bits16(X_bits)
    W_bits = bits16(W_bits)
    M, K = X_bits.shape
    Xf = bf16_to_f32(X_bits) if x_is_bf16 else f16_to_f32(X_bits)
    Wf = bf16_to_f32(W_bits) if w_is_bf16 else f16_to_f32(W_bits)
    m = np.abs(Xf.astype(np.float64)).sum(axis=0) / M
    logm = np.log(np.maximum(m, 1e-30))
    mu = logm.mean()
    Yref = gemm_f32(Xf, Wf).astype(np.float64)
    losses = np.empty(n_grid, np.float64)
    cand = []
    for j in range(n_grid):
        s = np.exp((j / n_grid) * (logm - mu)).astype(np.float32)
        s_inv = (np.float32(1) / s).astype(np.float32)
        q, sc, zr = quantize_weights(W_bits, s, group_size, symmetric, is_bf16=w_is_bf16)
        Xp = awq_scale_acts(X_bits, s_inv, x_is_bf16)
        Xp = bf16_to_f32(f32_to_bf16(Xp)) if x_is_bf16 else f16_to_f32(f32_to_f16(Xp))
        Yq = gemm_f32(Xp, dequant(q, sc, zr, group_size)).astype(np.float64)
        losses[j] = ((Yref - Yq) ** 2).sum()
        cand.append(s)
    best = int(np.argmin(losses))
    return best, losses, cand[best]


# ---- block-scaled 4-bit floating point (NVFP4, MXFP4) --------------------------------
def e2m1_to_f32(c):
    return float(lib().oracle_e2m1_to_f32(int(c)))


def f32_to_e2m1(x):
    return int(lib().oracle_f32_to_e2m1(float(x)))


def e4m3_to_f32(b):
    return float(lib().oracle_e4m3_to_f32(int(b)))


def f32_to_e4m3(x):
    return int(lib().oracle_f32_to_e4m3(float(x)))


def nvfp4_quantize(A_bits, is_bf16=False):
    """NVFP4 of A [R,K] ("Production Quantization: AWQ, GPTQ, GGUF K-quants, FP8,
    MXFP4/NVFP4", section "MXFP4 / NVFP4": a scale per block; block of 16, E4M3 block
    scales and the tensor scale are readings, stated in w4_oracle.c).
    Returns (codes uint8 [R,K], block scales uint8 [R,K/16], tensor scale fp32)."""
    A_bits = bits16(A_bits)
    R, K = A_bits.shape
    codes = np.empty((R, K), np.uint8)
    bs = np.empty((R, K // 16), np.uint8)
    gs = ctypes.c_float()
    if lib().oracle_nvfp4_quantize(_p(A_bits), int(is_bf16), R, K, _p(codes), _p(bs), ctypes.byref(gs)) != 0:
        raise ValueError("NVFP4 needs K % 16 == 0")
    return codes, bs, np.float32(gs.value)


def nvfp4_dequant(codes, bscale, gs):
    codes = _c(codes, np.uint8)
    bscale = _c(bscale, np.uint8)
    R, K = codes.shape
    out = np.empty((R, K), np.float64)
    lib().oracle_nvfp4_dequant(_p(codes), _p(bscale), float(gs), R, K, _p(out))
    return out


def mxfp4_quantize(A_bits, is_bf16=False):
    """MXFP4 of A [R,K] (same page and section; block of 32 and the E8M0 scale are
    readings).  Returns (codes uint8 [R,K], scale bytes uint8 [R,K/32])."""
    A_bits = bits16(A_bits)
    R, K = A_bits.shape
    codes = np.empty((R, K), np.uint8)
    es = np.empty((R, K // 32), np.uint8)
    if lib().oracle_mxfp4_quantize(_p(A_bits), int(is_bf16), R, K, _p(codes), _p(es)) != 0:
        raise ValueError("MXFP4 needs K % 32 == 0")
    return codes, es


def mxfp4_dequant(codes, escale):
    codes = _c(codes, np.uint8)
    escale = _c(escale, np.uint8)
    R, K = codes.shape
    out = np.empty((R, K), np.float64)
    lib().oracle_mxfp4_dequant(_p(codes), _p(escale), R, K, _p(out))
    return out
