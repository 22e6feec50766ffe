"""CPU oracle for the quantization hot path -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The CUDA
library never does, and this package never touches it: the two share no code.

The arithmetic lives in ``wq_oracle.c`` (plain single-threaded C11, built with
``-O2 -fno-fast-math -ffp-contract=off`` so that every fp32 operation is one
IEEE-754 operation with round-to-nearest-even).  This module only marshals
numpy arrays in and out of it; each wrapper names the passage of the source
pages that the C routine follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
          "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile ``wq_oracle.c`` into ``liboracle.so`` (gcc) if it is missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
        if not _lib.orc_rounding_mode_is_nearest():
            raise RuntimeError("oracle requires the FE_TONEAREST rounding mode")
    return _lib


_P = ctypes.c_void_p
_I = ctypes.c_int


def _declare(L):
    L.orc_half_to_float.argtypes = [ctypes.c_uint16]
    L.orc_half_to_float.restype = ctypes.c_float
    L.orc_float_to_half.argtypes = [ctypes.c_float]
    L.orc_float_to_half.restype = ctypes.c_uint16
    L.orc_rounding_mode_is_nearest.restype = _I
    L.orc_quantize_group_int4.argtypes = [_P, _I, _I, _I, _I, _P, _P, _P]
    L.orc_quantize_group_int4.restype = _I
    L.orc_dequant_int4.argtypes = [_P, _P, _P, _I, _I, _I, _P]
    L.orc_dequant_int4.restype = None
    L.orc_quantize_sym_rows.argtypes = [_P, _I, _I, _P, _I, _I, _P, _P]
    L.orc_quantize_sym_rows.restype = _I
    L.orc_smooth.argtypes = [_P, _I, _P, _I, _I, ctypes.c_double, _P]
    L.orc_smooth.restype = _I
    L.orc_matmul_w4a16_ref.argtypes = [_P, _I, _P, _P, _P, _I, _I, _I, _P, _I, _P, _P]
    L.orc_matmul_w4a16_ref.restype = None
    L.orc_matmul_w4a16_ref_bf16.argtypes = [_P, _I, _P, _P, _P, _I, _I, _I, _P, _I, _P, _P]
    L.orc_matmul_w4a16_ref_bf16.restype = None
    L.orc_bf16_to_float.argtypes = [ctypes.c_uint16]
    L.orc_bf16_to_float.restype = ctypes.c_float
    L.orc_matmul_w8a16_ref.argtypes = [_P, _I, _P, _P, _I, _I, _P, _I, _P, _P]
    L.orc_matmul_w8a16_ref.restype = None
    L.orc_gemm_w8a8_ref.argtypes = [_P, _P, _P, _P, _I, _I, _I, _P, _I, _P, _I, _P, _P, _P]
    L.orc_gemm_w8a8_ref.restype = _I
    L.orc_e4m3_to_float.argtypes = [ctypes.c_uint8]
    L.orc_e4m3_to_float.restype = ctypes.c_float
    L.orc_float_to_e4m3.argtypes = [ctypes.c_float]
    L.orc_float_to_e4m3.restype = ctypes.c_uint8
    L.orc_quantize_fp8_e4m3.argtypes = [_P, _I, _I, _I, _P, _P]
    L.orc_quantize_fp8_e4m3.restype = _I
    L.orc_gemm_fp8_ref.argtypes = [_P, _P, _I, _P, _P, _I, _I, _I, _I, _P, _I, _P, _I, _P, _P]
    L.orc_gemm_fp8_ref.restype = None
    L.orc_outlier_columns.argtypes = [_P, _I, _I, ctypes.c_float, _I, _P]
    L.orc_outlier_columns.restype = _I
    L.orc_llm_int8_ref.argtypes = [_P, _I, _I, _P, _P, _I, _P, _I, _P, _I, _P, _I, _P, _P, _P, _P]
    L.orc_llm_int8_ref.restype = _I
    L.orc_e2m1_to_float.argtypes = [ctypes.c_uint8]
    L.orc_e2m1_to_float.restype = ctypes.c_float
    L.orc_float_to_e2m1.argtypes = [ctypes.c_float]
    L.orc_float_to_e2m1.restype = ctypes.c_uint8
    L.orc_e8m0_to_float.argtypes = [ctypes.c_uint8]
    L.orc_e8m0_to_float.restype = ctypes.c_float
    L.orc_quantize_mxfp4.argtypes = [_P, _I, _I, _P, _P]
    L.orc_quantize_mxfp4.restype = _I
    L.orc_quantize_nvfp4.argtypes = [_P, _I, _I, _P, _P, _P]
    L.orc_quantize_nvfp4.restype = _I
    L.orc_gemm_fp4_ref.argtypes = [_I, _P, _P, ctypes.c_float, _P, _P, ctypes.c_float, _I, _I, _I, _P, _I, _P, _I,
                                   _P, _P]
    L.orc_gemm_fp4_ref.restype = None
    L.orc_hessian.argtypes = [_P, _I, _I, _P]
    L.orc_hessian.restype = None
    L.orc_gptq_hinv_chol.argtypes = [_P, _I, ctypes.c_double, _P]
    L.orc_gptq_hinv_chol.restype = _I
    L.orc_gptq.argtypes = [_P, _I, _I, _I, _P, _P, _P, _P]
    L.orc_gptq.restype = _I
    L.orc_awq.argtypes = [_P, _I, _I, _I, _P, _I, _P, _P, _I, _P, _P, _P, _P, _P]
    L.orc_awq.restype = _I


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _f16_bits(a: np.ndarray) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype == np.float16:
        return np.ascontiguousarray(a).view(np.uint16)
    if a.dtype == np.uint16:
        return np.ascontiguousarray(a)
    raise TypeError(f"expected float16 (or its uint16 bits), got {a.dtype}")


# --------------------------------------------------------------------------
# binary16 conversions (IEEE 754 definition)
# --------------------------------------------------------------------------
def half_to_float(bits: int) -> float:
    return float(lib().orc_half_to_float(int(bits)))


def float_to_half(x: float) -> int:
    return int(lib().orc_float_to_half(float(np.float32(x))))


# --------------------------------------------------------------------------
# INT4 asymmetric per-group ("Quantization Explained", Scale and Zero-Point;
# "Quantization from Scratch", round-to-nearest quantize())
# --------------------------------------------------------------------------
def quantize_group_int4(w: np.ndarray, group_size: int = 128):
    """Returns (qweight u32 [N, K/8], scales fp16 [N, K/g], qzeros u32 [N, ceil(K/g/8)])."""
    w = np.asarray(w)
    if w.ndim != 2:
        raise ValueError("w must be 2-D [N, K]")
    N, K = w.shape
    if w.dtype == np.float32:
        src, is16 = _c(w, np.float32), 0
    else:
        src, is16 = _f16_bits(w), 1
    G = K // group_size
    qw = np.zeros((N, K // 8), np.uint32)
    sc = np.zeros((N, G), np.uint16)
    qz = np.zeros((N, (G + 7) // 8), np.uint32)
    rc = lib().orc_quantize_group_int4(_ptr(src), is16, N, K, group_size, _ptr(qw), _ptr(sc), _ptr(qz))
    if rc != 0:
        raise ValueError(f"orc_quantize_group_int4: bad arguments N={N} K={K} g={group_size}")
    return qw, sc.view(np.float16), qz


def dequant_int4(qweight, scales, qzeros, K: int, group_size: int = 128) -> np.ndarray:
    """w^ = s (q - z) in fp64, [N, K] ("Quantization from Scratch", Scale and zero-point)."""
    qw = _c(qweight, np.uint32)
    sc = _f16_bits(scales)
    qz = _c(qzeros, np.uint32)
    N = qw.shape[0]
    out = np.zeros((N, K), np.float64)
    lib().orc_dequant_int4(_ptr(qw), _ptr(sc), _ptr(qz), N, K, group_size, _ptr(out))
    return out


def unpack_int4_codes(qweight, K: int) -> np.ndarray:
    """Codes q[n, k] in [0, 15] from the packed layout (nibble k mod 8 of word k/8)."""
    qw = _c(qweight, np.uint32)
    shifts = (4 * np.arange(8, dtype=np.uint32))
    codes = (qw[:, :, None] >> shifts[None, None, :]) & 0xF
    return codes.reshape(qw.shape[0], K).astype(np.int32)


def unpack_int4_zeros(qzeros, G: int) -> np.ndarray:
    qz = _c(qzeros, np.uint32)
    shifts = (4 * np.arange(8, dtype=np.uint32))
    z = (qz[:, :, None] >> shifts[None, None, :]) & 0xF
    return z.reshape(qz.shape[0], -1)[:, :G].astype(np.int32)


# --------------------------------------------------------------------------
# INT8 symmetric per row ("How quantization works": math, quant.py, q8_per_row,
# SmoothQuant Xs = X / s, Ws = W * s)
# --------------------------------------------------------------------------
def quantize_int8_per_channel(w: np.ndarray, smooth: np.ndarray | None = None):
    """Weights [N, K] fp16 -> (int8 [N, K], fp32 scales [N]); w*s_j first if smooth."""
    return quantize_sym_rows(w, smooth, 1, 8)


def quantize_int8_per_token(x: np.ndarray, smooth: np.ndarray | None = None):
    """Activations [M, K] fp16 -> (int8 [M, K], fp32 scales [M]); x/s_j first if smooth."""
    return quantize_sym_rows(x, smooth, 2, 8)


def quantize_sym_rows(a, smooth=None, mode: int = 0, bits: int = 8):
    """Symmetric b-bit quantization, one scale per row of ``a`` (fp16 [R, K]).
    mode 1 multiplies column k by smooth[k] first, mode 2 divides by it."""
    bits16 = _f16_bits(a)
    R, K = bits16.shape
    sm = None if smooth is None else _c(smooth, np.float32)
    if sm is not None and sm.shape != (K,):
        raise ValueError("smooth must have shape [K]")
    q = np.zeros((R, K), np.int8)
    s = np.zeros(R, np.float32)
    rc = lib().orc_quantize_sym_rows(_ptr(bits16), R, K, _ptr(sm), mode if sm is not None else 0,
                                     int(bits), _ptr(q), _ptr(s))
    if rc != 0:
        raise ValueError("orc_quantize_sym_rows: bad arguments")
    return q, s


def smooth_factors(x: np.ndarray, w: np.ndarray, alpha: float = 0.5) -> np.ndarray:
    """s_j = max|X_j|^a / max|W_j|^(1-a) ("How quantization works", SmoothQuant)."""
    xb, wb = _f16_bits(x), _f16_bits(w)
    M, K = xb.shape
    N, K2 = wb.shape
    if K != K2:
        raise ValueError("X and W must share K")
    s = np.zeros(K, np.float32)
    rc = lib().orc_smooth(_ptr(xb), M, _ptr(wb), N, K, float(alpha), _ptr(s))
    if rc != 0:
        raise ValueError("orc_smooth: bad arguments")
    return s


# --------------------------------------------------------------------------
# fp64 matmul references
# --------------------------------------------------------------------------
def _rows_arg(rows, N):
    if rows is None:
        return None, N
    r = _c(rows, np.int32)
    if r.size and (r.min() < 0 or r.max() >= N):
        raise ValueError("row index out of range")
    return r, int(r.size)


def matmul_w4a16_ref_bf16(x_bits, qweight, scales, qzeros, K: int, group_size: int = 128, rows=None):
    """matmul_w4a16_ref with bf16 activations given as uint16 bit patterns [B, K]."""
    xb = np.ascontiguousarray(np.atleast_2d(x_bits), dtype=np.uint16)
    B = xb.shape[0]
    qw = _c(qweight, np.uint32)
    sc = _f16_bits(scales)
    qz = _c(qzeros, np.uint32)
    N = qw.shape[0]
    r, nr = _rows_arg(rows, N)
    y = np.zeros((B, nr), np.float64)
    bd = np.zeros((B, nr), np.float64)
    lib().orc_matmul_w4a16_ref_bf16(_ptr(xb), B, _ptr(qw), _ptr(sc), _ptr(qz), N, K, group_size,
                                    _ptr(r), nr, _ptr(y), _ptr(bd))
    return y, bd


def bf16_to_float(bits: int) -> float:
    return float(lib().orc_bf16_to_float(int(bits)))


def matmul_w4a16_ref(x, qweight, scales, qzeros, K: int, group_size: int = 128, rows=None):
    """(y [B, nrows], bound [B, nrows]) in fp64: y = sum_k s(q-z) x, bound = sum_k |s(q-z) x|."""
    xb = _f16_bits(np.atleast_2d(x))
    B = xb.shape[0]
    qw = _c(qweight, np.uint32)
    sc = _f16_bits(scales)
    qz = _c(qzeros, np.uint32)
    N = qw.shape[0]
    r, nr = _rows_arg(rows, N)
    y = np.zeros((B, nr), np.float64)
    bd = np.zeros((B, nr), np.float64)
    lib().orc_matmul_w4a16_ref(_ptr(xb), B, _ptr(qw), _ptr(sc), _ptr(qz), N, K, group_size,
                               _ptr(r), nr, _ptr(y), _ptr(bd))
    return y, bd


def matmul_w8a16_ref(x, wq, sw, rows=None):
    xb = _f16_bits(np.atleast_2d(x))
    B, K = xb.shape
    q = _c(wq, np.int8)
    s = _c(sw, np.float32)
    N = q.shape[0]
    r, nr = _rows_arg(rows, N)
    y = np.zeros((B, nr), np.float64)
    bd = np.zeros((B, nr), np.float64)
    lib().orc_matmul_w8a16_ref(_ptr(xb), B, _ptr(q), _ptr(s), N, K, _ptr(r), nr, _ptr(y), _ptr(bd))
    return y, bd


def gemm_w8a8_ref(xq, sx, wq, sw, ms=None, ns=None):
    """(acc int64 [nm, nn], y fp64, bound fp64) on the selected rows of X (ms) and of W (ns)."""
    a = _c(xq, np.int8)
    b = _c(wq, np.int8)
    M, K = a.shape
    N = b.shape[0]
    sxa = _c(sx, np.float32)
    swa = _c(sw, np.float32)
    m_arr, nm = _rows_arg(ms, M)
    n_arr, nn = _rows_arg(ns, N)
    acc = np.zeros((nm, nn), np.int64)
    y = np.zeros((nm, nn), np.float64)
    bd = np.zeros((nm, nn), np.float64)
    rc = lib().orc_gemm_w8a8_ref(_ptr(a), _ptr(sxa), _ptr(b), _ptr(swa), M, N, K, _ptr(m_arr), nm,
                                 _ptr(n_arr), nn, _ptr(acc), _ptr(y), _ptr(bd))
    if rc == -2:
        raise OverflowError("an int8 accumulator left the int32 range")
    return acc, y, bd


# --------------------------------------------------------------------------
# FP8 E4M3 ("Quantization from Scratch", Formats; "Quantization: Smaller
# Weights, Same Answers (Mostly)", FP8 section; "How quantization works",
# quant.py fake_quant_fp8: scale = max|w| / 448)
# --------------------------------------------------------------------------
def e4m3_to_float(code: int) -> float:
    return float(lib().orc_e4m3_to_float(int(code) & 0xFF))


def float_to_e4m3(x: float) -> int:
    return int(lib().orc_float_to_e4m3(float(np.float32(x))))


def quantize_fp8_e4m3(a, per_row: bool = True):
    """fp16 [R, K] -> (E4M3 codes uint8 [R, K], fp32 scales [R] per row or [1] per tensor)."""
    bits16 = _f16_bits(a)
    R, K = bits16.shape
    q = np.zeros((R, K), np.uint8)
    s = np.zeros(R if per_row else 1, np.float32)
    rc = lib().orc_quantize_fp8_e4m3(_ptr(bits16), R, K, 1 if per_row else 0, _ptr(q), _ptr(s))
    if rc != 0:
        raise ValueError("orc_quantize_fp8_e4m3: bad arguments")
    return q, s


def gemm_fp8_ref(xq, sx, wq, sw, ms=None, ns=None):
    """(y fp64 [nm, nn], bound fp64): y = sx * sw * sum_k e4m3(xq) e4m3(wq); a scale vector of
    length 1 applies to every row of its operand (per-tensor scale)."""
    a = _c(xq, np.uint8)
    b = _c(wq, np.uint8)
    M, K = a.shape
    N = b.shape[0]
    sxa = _c(np.atleast_1d(sx), np.float32)
    swa = _c(np.atleast_1d(sw), np.float32)
    m_arr, nm = _rows_arg(ms, M)
    n_arr, nn = _rows_arg(ns, N)
    y = np.zeros((nm, nn), np.float64)
    bd = np.zeros((nm, nn), np.float64)
    lib().orc_gemm_fp8_ref(_ptr(a), _ptr(sxa), int(sxa.size == M), _ptr(b), _ptr(swa), int(swa.size == N),
                           M, N, K, _ptr(m_arr), nm, _ptr(n_arr), nn, _ptr(y), _ptr(bd))
    return y, bd


# --------------------------------------------------------------------------
# LLM.int8() decomposition ("Quantization" (engine-room ch. 15), The
# Mathematics: C ~= S_out (.) (X_q W_q) + X_16 W_16)
# --------------------------------------------------------------------------
def outlier_columns(x, threshold: float, cap: int):
    """(idx int32 [min(total, cap)], total): columns with max |x| >= threshold, lowest first."""
    xb = _f16_bits(x)
    M, K = xb.shape
    idx = np.zeros(max(1, cap), np.int32)
    total = lib().orc_outlier_columns(_ptr(xb), M, K, float(np.float32(threshold)), int(cap), _ptr(idx))
    return idx[: min(total, cap)].copy(), int(total)


def llm_int8_ref(x, wq, sw, idx, ms=None, ns=None):
    """(y fp64 [nm, nn], bound, xq int8 [M, K], sx fp32 [M]) of the decomposed product with the
    columns `idx` carved out of the INT8 path (weights: per-channel INT8 codes wq and scales sw)."""
    xb = _f16_bits(x)
    M, K = xb.shape
    q = _c(wq, np.int8)
    s = _c(sw, np.float32)
    N = q.shape[0]
    ix = _c(idx, np.int32)
    m_arr, nm = _rows_arg(ms, M)
    n_arr, nn = _rows_arg(ns, N)
    xq = np.zeros((M, K), np.int8)
    sx = np.zeros(M, np.float32)
    y = np.zeros((nm, nn), np.float64)
    bd = np.zeros((nm, nn), np.float64)
    rc = lib().orc_llm_int8_ref(_ptr(xb), M, K, _ptr(q), _ptr(s), N, _ptr(ix), int(ix.size), _ptr(m_arr), nm,
                                _ptr(n_arr), nn, _ptr(xq), _ptr(sx), _ptr(y), _ptr(bd))
    if rc != 0:
        raise ValueError("orc_llm_int8_ref: bad arguments")
    return y, bd, xq, sx


# --------------------------------------------------------------------------
# Block-scaled FP4: MXFP4 (E2M1, blocks of 32, E8M0 power-of-two scales) and
# NVFP4 (E2M1, blocks of 16, E4M3 scales, one fp32 tensor scale)
# ("Quantization: Smaller Weights, Same Answers (Mostly)", FP8/MXFP4/NVFP4
# section; "Quantization from Scratch", Formats)
# --------------------------------------------------------------------------
def e2m1_to_float(code: int) -> float:
    return float(lib().orc_e2m1_to_float(int(code) & 0xF))


def float_to_e2m1(x: float) -> int:
    return int(lib().orc_float_to_e2m1(float(np.float32(x))))


def e8m0_to_float(code: int) -> float:
    return float(lib().orc_e8m0_to_float(int(code) & 0xFF))


def quantize_mxfp4(a):
    """fp16 [R, K] -> (packed E2M1 uint8 [R, K/2], E8M0 scales uint8 [R, K/32])."""
    xb = _f16_bits(a)
    R, K = xb.shape
    q = np.zeros((R, K // 2), np.uint8)
    s = np.zeros((R, K // 32), np.uint8)
    if lib().orc_quantize_mxfp4(_ptr(xb), R, K, _ptr(q), _ptr(s)) != 0:
        raise ValueError("orc_quantize_mxfp4: bad arguments")
    return q, s


def quantize_nvfp4(a):
    """fp16 [R, K] -> (packed E2M1 uint8 [R, K/2], E4M3 scales uint8 [R, K/16], fp32 tensor scale [1])."""
    xb = _f16_bits(a)
    R, K = xb.shape
    q = np.zeros((R, K // 2), np.uint8)
    s = np.zeros((R, K // 16), np.uint8)
    t = np.zeros(1, np.float32)
    if lib().orc_quantize_nvfp4(_ptr(xb), R, K, _ptr(q), _ptr(s), _ptr(t)) != 0:
        raise ValueError("orc_quantize_nvfp4: bad arguments")
    return q, s, t


def unpack_fp4(q, K: int) -> np.ndarray:
    """E2M1 codes [R, K] from the packed layout (element 2i in the low nibble of byte i)."""
    q = _c(q, np.uint8)
    out = np.empty((q.shape[0], K), np.uint8)
    out[:, 0::2] = q & 0xF
    out[:, 1::2] = q >> 4
    return out


def gemm_fp4_ref(nvfp4: bool, a, sa, ta, b, sb, tb, K: int, ms=None, ns=None):
    """(y fp64, bound) of the block-scaled FP4 product (tensor scales ta/tb: 1.0 for MXFP4)."""
    A, SA, B, SB = _c(a, np.uint8), _c(sa, np.uint8), _c(b, np.uint8), _c(sb, np.uint8)
    M, N = A.shape[0], B.shape[0]
    m_arr, nm = _rows_arg(ms, M)
    n_arr, nn = _rows_arg(ns, N)
    y = np.zeros((nm, nn), np.float64)
    bd = np.zeros((nm, nn), np.float64)
    lib().orc_gemm_fp4_ref(1 if nvfp4 else 0, _ptr(A), _ptr(SA), float(ta), _ptr(B), _ptr(SB), float(tb), M, N, K,
                           _ptr(m_arr), nm, _ptr(n_arr), nn, _ptr(y), _ptr(bd))
    return y, bd


# --------------------------------------------------------------------------
# Calibration-driven INT4 ("Quantization from Scratch": GPTQ, AWQ, gptq()/awq()
# in "Measured on two real layers"; "Quantization" (engine-room ch. 15): H = 2 X^T X)
# --------------------------------------------------------------------------
def hessian(x) -> np.ndarray:
    """H = 2 X^T X in fp64 from fp16 calibration activations X [T, K]."""
    xb = _f16_bits(x)
    T, K = xb.shape
    H = np.zeros((K, K), np.float64)
    lib().orc_hessian(_ptr(xb), T, K, _ptr(H))
    return H


def gptq_hinv_chol(H, damp: float = 0.01) -> np.ndarray:
    """U, upper triangular with U^T U = (H + damp * mean(diag H) I)^-1."""
    Hc = _c(H, np.float64)
    K = Hc.shape[0]
    U = np.zeros((K, K), np.float64)
    if lib().orc_gptq_hinv_chol(_ptr(Hc), K, float(damp), _ptr(U)) != 0:
        raise ValueError("H + damping is not positive definite")
    return U


def gptq(w, U, group_size: int = 128):
    """GPTQ in the stored INT4 format: (qweight u32 [N, K/8], scales fp16 [N, K/g], qzeros u32)."""
    wb = _f16_bits(w)
    N, K = wb.shape
    Uc = _c(U, np.float64)
    G = K // group_size
    qw = np.zeros((N, K // 8), np.uint32)
    sc = np.zeros((N, G), np.uint16)
    qz = np.zeros((N, (G + 7) // 8), np.uint32)
    if lib().orc_gptq(_ptr(wb), N, K, group_size, _ptr(Uc), _ptr(qw), _ptr(sc), _ptr(qz)) != 0:
        raise ValueError("orc_gptq: bad arguments")
    return qw, sc.view(np.float16), qz


AWQ_GRID = np.linspace(0.0, 1.0, 11)


def awq(w, x, H, group_size: int = 128, grid=AWQ_GRID):
    """AWQ's scaling search: (qweight, scales, qzeros of W diag(s), s fp32 [K], alpha index, errors)."""
    wb, xb = _f16_bits(w), _f16_bits(x)
    N, K = wb.shape
    T = xb.shape[0]
    Hc = _c(H, np.float64)
    gr = _c(grid, np.float64)
    G = K // group_size
    qw = np.zeros((N, K // 8), np.uint32)
    sc = np.zeros((N, G), np.uint16)
    qz = np.zeros((N, (G + 7) // 8), np.uint32)
    s = np.zeros(K, np.float32)
    err = np.zeros(gr.size, np.float64)
    best = lib().orc_awq(_ptr(wb), N, K, group_size, _ptr(xb), T, _ptr(Hc), _ptr(gr), int(gr.size), _ptr(qw),
                         _ptr(sc), _ptr(qz), _ptr(s), _ptr(err))
    if best < 0:
        raise ValueError("orc_awq: bad arguments")
    return qw, sc.view(np.float16), qz, s, int(best), err
