"""Python binding of ``libwq.so``, the sm_100a weight/activation quantization library.

Argument marshalling only: every function checks tensor devices, dtypes and
shapes, allocates outputs with PyTorch (PyTorch owns device memory and streams
here), and calls the C entry point of the same name on the current CUDA stream.
All arithmetic runs in the library's kernels.  There is no CPU fallback: if
``libwq.so`` is missing the import fails.

Packed INT4 tensors are carried as ``torch.int32`` (bit-identical to the
library's ``uint32`` words) and fp16 as ``torch.float16``.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["WQError", "lib", "quantize_group_int4", "quantize_int8_per_channel", "quantize_int8_per_token",
           "smooth", "smooth_workspace_bytes", "smooth_noalloc", "gemv_w4a16", "gemm_w4a16", "gemm_w8a8", "gemv_w8a16",
           "matmul_w4a16", "quantize_fp8_e4m3", "gemm_fp8", "outlier_columns", "gather_outliers",
           "gemm_w8a8_outliers", "llm_int8_matmul", "quantize_mxfp4", "quantize_nvfp4", "gemm_fp4",
           "gemv_w4a16_bf16", "gemm_w4a16_bf16", "hessian", "gptq_prepare", "gptq_quantize", "awq", "device_status", "set_wait_limit",
           "selftest_wait_timeout", "LIB_PATH"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libwq.so")

WQ_OK, WQ_ERR_INVALID_ARG, WQ_ERR_ALIGNMENT, WQ_ERR_UNSUPPORTED, WQ_ERR_CUDA, WQ_ERR_TIMEOUT = range(6)
WQ_F32, WQ_F16 = 0, 1
_STATUS = {0: "WQ_OK", 1: "WQ_ERR_INVALID_ARG", 2: "WQ_ERR_ALIGNMENT", 3: "WQ_ERR_UNSUPPORTED",
           4: "WQ_ERR_CUDA", 5: "WQ_ERR_TIMEOUT"}


class WQError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {_STATUS.get(status, status)}: {message}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python bit_gemv_gemm_group_b200/build.py`")

lib = ctypes.CDLL(LIB_PATH)

_P, _I, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
_SIGS = {
    "wq_quantize_group_int4": [_P, _I, _I, _I, _I, _P, _P, _P, _P],
    "wq_quantize_int8_per_channel": [_P, _I, _I, _P, _P, _P, _P],
    "wq_quantize_int8_per_token": [_P, _I, _I, _P, _P, _P, _P],
    "wq_smooth": [_P, _I, _P, _I, _I, _F, _P, _P, _P],
    "wq_smooth_noalloc": [_P, _I, _P, _I, _I, _F, _P, _P],
    "wq_gemv_w4a16": [_P, _I, _P, _P, _P, _I, _I, _I, _P, _P],
    "wq_gemm_w4a16": [_P, _I, _P, _P, _P, _I, _I, _I, _P, _P],
    "wq_gemm_w8a8": [_P, _P, _P, _P, _I, _I, _I, _P, _P, _P],
    "wq_gemv_w8a16": [_P, _I, _P, _P, _I, _I, _P, _P],
    "wq_quantize_fp8_e4m3": [_P, _I, _I, _I, _P, _P, _P],
    "wq_gemm_fp8": [_P, _P, _I, _P, _P, _I, _I, _I, _I, _P, _P, _P],
    "wq_outlier_columns": [_P, _I, _I, _F, _I, _P, _P, _P, _P],
    "wq_gather_outliers": [_P, _I, _I, _P, _I, _P, _P, _I, _P, _P, _P],
    "wq_gemm_w8a8_outliers": [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P],
    "wq_quantize_mxfp4": [_P, _I, _I, _P, _P, _P],
    "wq_quantize_nvfp4": [_P, _I, _I, _P, _P, _P, _P],
    "wq_gemm_fp4": [_I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P],
    "wq_hessian": [_P, _I, _I, _P, _P],
    "wq_gemv_w4a16_bf16": [_P, _I, _P, _P, _P, _I, _I, _I, _P, _P],
    "wq_gemm_w4a16_bf16": [_P, _I, _P, _P, _P, _I, _I, _I, _P, _P],
    "wq_gptq_prepare": [_P, _I, _F, _P, _P, _P],
    "wq_gptq_quantize": [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P],
    "wq_awq": [_P, _I, _I, _I, _P, _I, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P],
    "wq_device_status": [_P],
    "wq_selftest_wait_timeout": [_P],
}
for _name, _args in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.argtypes = _args
    _fn.restype = ctypes.c_int
lib.wq_last_error.argtypes = []
lib.wq_last_error.restype = ctypes.c_char_p
lib.wq_smooth_workspace_bytes.argtypes = [_I]
lib.wq_smooth_workspace_bytes.restype = ctypes.c_size_t
lib.wq_gptq_workspace_bytes.argtypes = [_I]
lib.wq_gptq_workspace_bytes.restype = ctypes.c_size_t
lib.wq_fp4_scale_bytes.argtypes = [_I, _I, _I]
lib.wq_fp4_scale_bytes.restype = ctypes.c_size_t
lib.wq_awq_workspace_bytes.argtypes = [_I, _I]
lib.wq_awq_workspace_bytes.restype = ctypes.c_size_t
lib.wq_set_wait_limit.argtypes = [ctypes.c_uint64]
lib.wq_set_wait_limit.restype = None


def _check(status: int, where: str):
    if status != WQ_OK:
        raise WQError(status, where, lib.wq_last_error().decode(errors="replace"))


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _cuda(t: torch.Tensor, name: str, dtypes, ndim=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-D, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _empty(shape, dtype, like: torch.Tensor) -> torch.Tensor:
    return torch.empty(shape, dtype=dtype, device=like.device)


# --------------------------------------------------------------------------
# quantizers
# --------------------------------------------------------------------------
def quantize_group_int4(w: torch.Tensor, group_size: int = 128, stream=None):
    """Asymmetric INT4 per group -> (qweight int32 [N, K/8], scales fp16 [N, K/g], qzeros int32 [N, ceil(K/g/8)])."""
    _cuda(w, "w", (torch.float16, torch.float32), 2)
    N, K = w.shape
    G = K // group_size if group_size > 0 else 0
    qw = _empty((N, K // 8), torch.int32, w)
    sc = _empty((N, G), torch.float16, w)
    qz = _empty((N, (G + 7) // 8), torch.int32, w)
    dt = WQ_F16 if w.dtype == torch.float16 else WQ_F32
    _check(lib.wq_quantize_group_int4(_ptr(w), dt, N, K, group_size, _ptr(qw), _ptr(sc), _ptr(qz),
                                      _P(_stream(stream))), "wq_quantize_group_int4")
    return qw, sc, qz


def _q8(fn, name, a, smooth_vec, stream):
    _cuda(a, "input", (torch.float16,), 2)
    R, K = a.shape
    if smooth_vec is not None:
        _cuda(smooth_vec, "smooth", (torch.float32,), 1)
        if smooth_vec.numel() != K:
            raise ValueError("smooth must have K elements")
    q = _empty((R, K), torch.int8, a)
    s = _empty((R,), torch.float32, a)
    _check(fn(_ptr(a), R, K, _ptr(smooth_vec), _ptr(q), _ptr(s), _P(_stream(stream))), name)
    return q, s


def quantize_int8_per_channel(w: torch.Tensor, smooth_vec: torch.Tensor | None = None, stream=None):
    """Symmetric INT8 per row of weights (w * s_j first when smoothing) -> (int8 [N, K], fp32 [N])."""
    return _q8(lib.wq_quantize_int8_per_channel, "wq_quantize_int8_per_channel", w, smooth_vec, stream)


def quantize_int8_per_token(x: torch.Tensor, smooth_vec: torch.Tensor | None = None, stream=None):
    """Symmetric INT8 per activation row (x / s_j first when smoothing) -> (int8 [M, K], fp32 [M])."""
    return _q8(lib.wq_quantize_int8_per_token, "wq_quantize_int8_per_token", x, smooth_vec, stream)


def smooth_workspace_bytes(K: int) -> int:
    return int(lib.wq_smooth_workspace_bytes(int(K)))


def smooth(x: torch.Tensor, w: torch.Tensor, alpha: float = 0.5, workspace: torch.Tensor | None = None,
           stream=None) -> torch.Tensor:
    """SmoothQuant factors s_j = max|X_j|^alpha / max|W_j|^(1-alpha) -> fp32 [K]."""
    _cuda(x, "x", (torch.float16,), 2)
    _cuda(w, "w", (torch.float16,), 2)
    M, K = x.shape
    N, K2 = w.shape
    if K != K2:
        raise ValueError("x and w must share K")
    s = _empty((K,), torch.float32, x)
    if workspace is None:
        workspace = _empty((max(1, smooth_workspace_bytes(K)),), torch.uint8, x)
    _cuda(workspace, "workspace", (torch.uint8,), 1)
    if workspace.numel() < smooth_workspace_bytes(K):
        raise ValueError("workspace too small")
    _check(lib.wq_smooth(_ptr(x), M, _ptr(w), N, K, float(alpha), _ptr(s), _ptr(workspace), _P(_stream(stream))),
           "wq_smooth")
    return s


SMOOTH_NOALLOC_MAX_K = 65536


def smooth_noalloc(x: torch.Tensor, w: torch.Tensor, alpha: float = 0.5, s: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """`smooth` through the entry point that allocates no device memory in the library call.

    The workspace is the library's built-in device array (K <= SMOOTH_NOALLOC_MAX_K); pass `s`
    (fp32 [K], on x's device) to keep this wrapper allocation-free as well.  Calls that overlap
    on the GPU share that array and race."""
    _cuda(x, "x", (torch.float16,), 2)
    _cuda(w, "w", (torch.float16,), 2)
    M, K = x.shape
    N, K2 = w.shape
    if K != K2:
        raise ValueError("x and w must share K")
    if s is None:
        s = _empty((K,), torch.float32, x)
    _cuda(s, "s", (torch.float32,), 1)
    if s.numel() != K:
        raise ValueError("s must have K elements")
    _check(lib.wq_smooth_noalloc(_ptr(x), M, _ptr(w), N, K, float(alpha), _ptr(s), _P(_stream(stream))),
           "wq_smooth_noalloc")
    return s


# --------------------------------------------------------------------------
# matmuls
# --------------------------------------------------------------------------
def _w4_args(x, qweight, scales, qzeros, group_size, xdtype=torch.float16):
    _cuda(x, "x", (xdtype,), 2)
    _cuda(qweight, "qweight", (torch.int32,), 2)
    _cuda(scales, "scales", (torch.float16,), 2)
    _cuda(qzeros, "qzeros", (torch.int32,), 2)
    B, K = x.shape
    N = qweight.shape[0]
    if qweight.shape[1] * 8 != K:
        raise ValueError("qweight must be [N, K/8]")
    if group_size <= 0 or K % group_size or tuple(scales.shape) != (N, K // group_size):
        raise ValueError("scales must be [N, K/group_size]")
    if tuple(qzeros.shape) != (N, (K // group_size + 7) // 8):
        raise ValueError("qzeros must be [N, ceil(K/group_size/8)]")
    return B, N, K


def gemv_w4a16(x, qweight, scales, qzeros, group_size: int = 128, out=None, stream=None):
    """y [B, N] fp16 = x [B, K] @ dequant(W)^T for B = 1..8 (fused dequant GEMV)."""
    B, N, K = _w4_args(x, qweight, scales, qzeros, group_size)
    y = out if out is not None else _empty((B, N), torch.float16, x)
    _cuda(y, "out", (torch.float16,), 2)
    _check(lib.wq_gemv_w4a16(_ptr(x), B, _ptr(qweight), _ptr(scales), _ptr(qzeros), N, K, group_size, _ptr(y),
                             _P(_stream(stream))), "wq_gemv_w4a16")
    return y


def gemm_w4a16(x, qweight, scales, qzeros, group_size: int = 128, out=None, stream=None):
    """y [M, N] fp16 = x [M, K] @ dequant(W)^T for M >= 16 (or 9..15 with K % 256 == 0)."""
    M, N, K = _w4_args(x, qweight, scales, qzeros, group_size)
    y = out if out is not None else _empty((M, N), torch.float16, x)
    _cuda(y, "out", (torch.float16,), 2)
    _check(lib.wq_gemm_w4a16(_ptr(x), M, _ptr(qweight), _ptr(scales), _ptr(qzeros), N, K, group_size, _ptr(y),
                             _P(_stream(stream))), "wq_gemm_w4a16")
    return y


def gemv_w4a16_bf16(x, qweight, scales, qzeros, group_size: int = 128, out=None, stream=None):
    """bf16 y [B, N] = x [B, K] (bf16) @ dequant(W)^T for B = 1..8."""
    B, N, K = _w4_args(x, qweight, scales, qzeros, group_size, torch.bfloat16)
    y = out if out is not None else _empty((B, N), torch.bfloat16, x)
    _cuda(y, "out", (torch.bfloat16,), 2)
    _check(lib.wq_gemv_w4a16_bf16(_ptr(x), B, _ptr(qweight), _ptr(scales), _ptr(qzeros), N, K, group_size, _ptr(y),
                                  _P(_stream(stream))), "wq_gemv_w4a16_bf16")
    return y


def gemm_w4a16_bf16(x, qweight, scales, qzeros, group_size: int = 128, out=None, stream=None):
    """bf16 y [M, N] = x [M, K] (bf16) @ dequant(W)^T for M >= 9."""
    M, N, K = _w4_args(x, qweight, scales, qzeros, group_size, torch.bfloat16)
    y = out if out is not None else _empty((M, N), torch.bfloat16, x)
    _cuda(y, "out", (torch.bfloat16,), 2)
    _check(lib.wq_gemm_w4a16_bf16(_ptr(x), M, _ptr(qweight), _ptr(scales), _ptr(qzeros), N, K, group_size, _ptr(y),
                                  _P(_stream(stream))), "wq_gemm_w4a16_bf16")
    return y


def matmul_w4a16(x, qweight, scales, qzeros, group_size: int = 128, out=None, stream=None):
    """GEMV for up to 8 activation rows, GEMM above (the caller's choice made for it)."""
    if x.shape[0] <= 8:
        return gemv_w4a16(x, qweight, scales, qzeros, group_size, out, stream)
    return gemm_w4a16(x, qweight, scales, qzeros, group_size, out, stream)


def gemm_w8a8(xq, sx, wq, sw, out=None, return_acc: bool = False, acc_out=None, stream=None):
    """y [M, N] fp16 = fp16((xq @ wq^T) * sx[m] * sw[n]); optionally also the int32 accumulators."""
    _cuda(xq, "xq", (torch.int8,), 2)
    _cuda(wq, "wq", (torch.int8,), 2)
    _cuda(sx, "sx", (torch.float32,), 1)
    _cuda(sw, "sw", (torch.float32,), 1)
    M, K = xq.shape
    N, K2 = wq.shape
    if K != K2 or sx.numel() != M or sw.numel() != N:
        raise ValueError("shape mismatch: xq [M,K], wq [N,K], sx [M], sw [N]")
    y = out if out is not None else _empty((M, N), torch.float16, xq)
    _cuda(y, "out", (torch.float16,), 2)
    acc = acc_out
    if acc is None and return_acc:
        acc = _empty((M, N), torch.int32, xq)
    if acc is not None:
        _cuda(acc, "acc_out", (torch.int32,), 2)
    _check(lib.wq_gemm_w8a8(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), M, N, K, _ptr(y), _ptr(acc),
                            _P(_stream(stream))), "wq_gemm_w8a8")
    return (y, acc) if (return_acc or acc_out is not None) else y


def gemv_w8a16(x, wq, sw, out=None, stream=None):
    """y [B, N] fp16 = fp16(sw[n] * (x @ wq^T)) for B = 1..8."""
    _cuda(x, "x", (torch.float16,), 2)
    _cuda(wq, "wq", (torch.int8,), 2)
    _cuda(sw, "sw", (torch.float32,), 1)
    B, K = x.shape
    N = wq.shape[0]
    if wq.shape[1] != K or sw.numel() != N:
        raise ValueError("shape mismatch: x [B,K], wq [N,K], sw [N]")
    y = out if out is not None else _empty((B, N), torch.float16, x)
    _cuda(y, "out", (torch.float16,), 2)
    _check(lib.wq_gemv_w8a16(_ptr(x), B, _ptr(wq), _ptr(sw), N, K, _ptr(y), _P(_stream(stream))), "wq_gemv_w8a16")
    return y


def quantize_fp8_e4m3(a: torch.Tensor, per_row: bool = True, stream=None):
    """FP8 E4M3 codes (torch.uint8 [R, K]) and fp32 scales ([R] per row, [1] per tensor) of fp16 `a`."""
    _cuda(a, "input", (torch.float16,), 2)
    R, K = a.shape
    q = _empty((R, K), torch.uint8, a)
    s = _empty((R if per_row else 1,), torch.float32, a)
    _check(lib.wq_quantize_fp8_e4m3(_ptr(a), R, K, 1 if per_row else 0, _ptr(q), _ptr(s), _P(_stream(stream))),
           "wq_quantize_fp8_e4m3")
    return q, s


def gemm_fp8(xq, sx, wq, sw, out=None, return_acc: bool = False, stream=None):
    """y [M, N] fp16 = fp16((e4m3(xq) @ e4m3(wq)^T) * sx * sw); a scale tensor of one element is per tensor."""
    _cuda(xq, "xq", (torch.uint8,), 2)
    _cuda(wq, "wq", (torch.uint8,), 2)
    _cuda(sx, "sx", (torch.float32,), 1)
    _cuda(sw, "sw", (torch.float32,), 1)
    M, K = xq.shape
    N, K2 = wq.shape
    if K != K2 or sx.numel() not in (1, M) or sw.numel() not in (1, N):
        raise ValueError("shape mismatch: xq [M,K], wq [N,K], sx [M] or [1], sw [N] or [1]")
    y = out if out is not None else _empty((M, N), torch.float16, xq)
    _cuda(y, "out", (torch.float16,), 2)
    acc = _empty((M, N), torch.float32, xq) if return_acc else None
    _check(lib.wq_gemm_fp8(_ptr(xq), _ptr(sx), int(sx.numel() == M), _ptr(wq), _ptr(sw), int(sw.numel() == N),
                           M, N, K, _ptr(y), _ptr(acc), _P(_stream(stream))), "wq_gemm_fp8")
    return (y, acc) if return_acc else y


def outlier_columns(x: torch.Tensor, threshold: float = 6.0, cap: int = 64, stream=None):
    """LLM.int8() outlier columns of fp16 x [M, K]: (idx int32 [cap], count int32 [1], keep fp32 [K]).

    idx[:min(count, cap)] are the carved columns (lowest first); keep is 0 there and 1 elsewhere."""
    _cuda(x, "x", (torch.float16,), 2)
    M, K = x.shape
    idx = _empty((cap,), torch.int32, x)  # the call writes every entry (0 past the carved ones)
    count = _empty((1,), torch.int32, x)
    keep = _empty((K,), torch.float32, x)
    _check(lib.wq_outlier_columns(_ptr(x), M, K, float(threshold), int(cap), _ptr(idx), _ptr(count), _ptr(keep),
                                  _P(_stream(stream))), "wq_outlier_columns")
    return idx, count, keep


def gather_outliers(x, wq, idx, count, cap: int, stream=None):
    """(X_16 fp16 [M, cap], W_16 fp16 [N, cap]): the carved columns of x and of the INT8 weight codes."""
    _cuda(x, "x", (torch.float16,), 2)
    _cuda(wq, "wq", (torch.int8,), 2)
    _cuda(idx, "idx", (torch.int32,), 1)
    _cuda(count, "count", (torch.int32,), 1)
    M, K = x.shape
    N = wq.shape[0]
    if wq.shape[1] != K or idx.numel() < cap:
        raise ValueError("shape mismatch: x [M,K], wq [N,K], idx [>= cap]")
    x16 = _empty((M, cap), torch.float16, x)
    w16 = _empty((N, cap), torch.float16, x)
    _check(lib.wq_gather_outliers(_ptr(x), M, K, _ptr(wq), N, _ptr(idx), _ptr(count), int(cap), _ptr(x16), _ptr(w16),
                                  _P(_stream(stream))), "wq_gather_outliers")
    return x16, w16


def gemm_w8a8_outliers(xq, sx, wq, sw, x16, w16, out=None, stream=None):
    """y [M, N] fp16 = fp16((xq @ wq^T * sx[m] + x16 @ w16^T) * sw[n]) (LLM.int8() product)."""
    for t, n, d in ((xq, "xq", torch.int8), (wq, "wq", torch.int8), (sx, "sx", torch.float32),
                    (sw, "sw", torch.float32), (x16, "x16", torch.float16), (w16, "w16", torch.float16)):
        _cuda(t, n, (d,))
    M, K = xq.shape
    N = wq.shape[0]
    cap = x16.shape[1]
    if wq.shape[1] != K or sx.numel() != M or sw.numel() != N or tuple(x16.shape) != (M, cap) or \
            tuple(w16.shape) != (N, cap):
        raise ValueError("shape mismatch: xq [M,K], wq [N,K], sx [M], sw [N], x16 [M,cap], w16 [N,cap]")
    y = out if out is not None else _empty((M, N), torch.float16, xq)
    _cuda(y, "out", (torch.float16,), 2)
    _check(lib.wq_gemm_w8a8_outliers(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), _ptr(x16), _ptr(w16), int(cap), M, N, K,
                                     _ptr(y), _P(_stream(stream))), "wq_gemm_w8a8_outliers")
    return y


def llm_int8_matmul(x, wq, sw, threshold: float = 6.0, cap: int = 64, stream=None):
    """The LLM.int8() sequence on fp16 x [M, K] and per-channel INT8 weights (wq [N, K], sw [N]):
    outlier columns -> per-token INT8 of the rest -> gather -> GEMM.  Returns (y, count)."""
    idx, count, keep = outlier_columns(x, threshold, cap, stream)
    xq, sx = quantize_int8_per_channel(x, keep, stream)
    x16, w16 = gather_outliers(x, wq, idx, count, cap, stream)
    return gemm_w8a8_outliers(xq, sx, wq, sw, x16, w16, stream=stream), count


def fp4_scale_bytes(R: int, K: int, nvfp4: bool) -> int:
    """Bytes of the scale-factor buffer of an R x K FP4 tensor (the tensor-core atom layout)."""
    return int(lib.wq_fp4_scale_bytes(int(R), int(K), 1 if nvfp4 else 0))


def quantize_mxfp4(x: torch.Tensor, stream=None):
    """MXFP4 of fp16 x [R, K]: (packed E2M1 codes uint8 [R, K/2], E8M0 scales uint8 in the atom layout)."""
    _cuda(x, "x", (torch.float16,), 2)
    R, K = x.shape
    q = _empty((R, K // 2), torch.uint8, x)
    s = _empty((fp4_scale_bytes(R, K, False),), torch.uint8, x)
    _check(lib.wq_quantize_mxfp4(_ptr(x), R, K, _ptr(q), _ptr(s), _P(_stream(stream))), "wq_quantize_mxfp4")
    return q, s


def quantize_nvfp4(x: torch.Tensor, stream=None):
    """NVFP4 of fp16 x [R, K]: (packed E2M1 uint8 [R, K/2], E4M3 scales uint8 in the atom layout,
    fp32 tensor scale [1])."""
    _cuda(x, "x", (torch.float16,), 2)
    R, K = x.shape
    q = _empty((R, K // 2), torch.uint8, x)
    s = _empty((fp4_scale_bytes(R, K, True),), torch.uint8, x)
    t = _empty((1,), torch.float32, x)
    _check(lib.wq_quantize_nvfp4(_ptr(x), R, K, _ptr(q), _ptr(s), _ptr(t), _P(_stream(stream))),
           "wq_quantize_nvfp4")
    return q, s, t


def gemm_fp4(a, sfa, b, sfb, ta=None, tb=None, out=None, return_acc: bool = False, stream=None):
    """Block-scaled FP4 GEMM: NVFP4 when the tensor scales ta/tb are given, MXFP4 otherwise.
    a [M, K/2], b [N, K/2] codes; sfa, sfb scale bytes in the atom layout -> y fp16 [M, N]."""
    nv = ta is not None
    for t, n in ((a, "a"), (b, "b")):
        _cuda(t, n, (torch.uint8,), 2)
    for t, n in ((sfa, "sfa"), (sfb, "sfb")):
        _cuda(t, n, (torch.uint8,), 1)
    if nv:
        _cuda(ta, "ta", (torch.float32,), 1)
        _cuda(tb, "tb", (torch.float32,), 1)
    M, K = a.shape[0], a.shape[1] * 2
    N = b.shape[0]
    if b.shape[1] * 2 != K or sfa.numel() != fp4_scale_bytes(M, K, nv) or sfb.numel() != fp4_scale_bytes(N, K, nv):
        raise ValueError("shape mismatch: a [M,K/2], b [N,K/2], sfa/sfb of fp4_scale_bytes(M or N, K) bytes")
    y = out if out is not None else _empty((M, N), torch.float16, a)
    _cuda(y, "out", (torch.float16,), 2)
    acc = _empty((M, N), torch.float32, a) if return_acc else None
    _check(lib.wq_gemm_fp4(1 if nv else 0, _ptr(a), _ptr(sfa), _ptr(ta), _ptr(b), _ptr(sfb), _ptr(tb), M, N, K,
                           _ptr(y), _ptr(acc), _P(_stream(stream))), "wq_gemm_fp4")
    return (y, acc) if return_acc else y


def hessian(x: torch.Tensor, stream=None) -> torch.Tensor:
    """H = 2 X^T X (fp32 [K, K]) from fp16 calibration activations x [T, K]."""
    _cuda(x, "x", (torch.float16,), 2)
    T, K = x.shape
    H = _empty((K, K), torch.float32, x)
    _check(lib.wq_hessian(_ptr(x), T, K, _ptr(H), _P(_stream(stream))), "wq_hessian")
    return H


def gptq_prepare(H: torch.Tensor, damp: float = 0.01, stream=None) -> torch.Tensor:
    """U (fp32 [K, K], upper) with U^T U = (H + damp * mean(diag H) I)^-1."""
    _cuda(H, "H", (torch.float32,), 2)
    K = H.shape[0]
    U = _empty((K, K), torch.float32, H)
    ws = _empty((max(16, int(lib.wq_gptq_workspace_bytes(K))),), torch.uint8, H)
    _check(lib.wq_gptq_prepare(_ptr(H), K, float(damp), _ptr(U), _ptr(ws), _P(_stream(stream))), "wq_gptq_prepare")
    return U


def gptq_quantize(w: torch.Tensor, U: torch.Tensor, group_size: int = 128, stream=None):
    """GPTQ of fp16 w [N, K] given U -> (qweight int32 [N, K/8], scales fp16 [N, K/g], qzeros int32)."""
    _cuda(w, "w", (torch.float16,), 2)
    _cuda(U, "U", (torch.float32,), 2)
    N, K = w.shape
    G = K // group_size
    work = _empty((N * K + N * 128,), torch.float32, w)
    qw = _empty((N, K // 8), torch.int32, w)
    sc = _empty((N, G), torch.float16, w)
    qz = _empty((N, (G + 7) // 8), torch.int32, w)
    _check(lib.wq_gptq_quantize(_ptr(w), N, K, group_size, _ptr(U), _ptr(work), _ptr(qw), _ptr(sc), _ptr(qz),
                                _P(_stream(stream))), "wq_gptq_quantize")
    return qw, sc, qz


def awq(w: torch.Tensor, x: torch.Tensor, grid=None, group_size: int = 128, stream=None):
    """AWQ's scaling search -> (qweight, scales, qzeros of W diag(s), s fp32 [K], err fp64 [len(grid)], best int32 [1])."""
    _cuda(w, "w", (torch.float16,), 2)
    _cuda(x, "x", (torch.float16,), 2)
    N, K = w.shape
    T = x.shape[0]
    g = [i / 10 for i in range(11)] if grid is None else [float(a) for a in grid]
    garr = (ctypes.c_double * len(g))(*g)
    G = K // group_size
    qw = _empty((N, K // 8), torch.int32, w)
    sc = _empty((N, G), torch.float16, w)
    qz = _empty((N, (G + 7) // 8), torch.int32, w)
    s = _empty((K,), torch.float32, w)
    err = _empty((len(g),), torch.float64, w)
    best = _empty((1,), torch.int32, w)
    ws = _empty((max(16, int(lib.wq_awq_workspace_bytes(N, K))),), torch.uint8, w)
    _check(lib.wq_awq(_ptr(w), N, K, group_size, _ptr(x), T, garr, len(g), _ptr(qw), _ptr(sc), _ptr(qz), _ptr(s),
                      _ptr(err), _ptr(best), _ptr(ws), _P(_stream(stream))), "wq_awq")
    return qw, sc, qz, s, err, best


def device_status(stream=None) -> int:
    """Synchronizes the stream and returns (and clears) the device status word (0 = WQ_OK)."""
    return int(lib.wq_device_status(_P(_stream(stream))))


def selftest_wait_timeout(stream=None) -> None:
    """Launches the bounded-wait self-test (a wait that must time out; see wq.h)."""
    _check(lib.wq_selftest_wait_timeout(_P(_stream(stream))), "wq_selftest_wait_timeout")


def set_wait_limit(nanoseconds: int) -> None:
    """Wall-clock limit of each bounded wait in the pipelined kernels (0 restores the 2 s default)."""
    lib.wq_set_wait_limit(int(nanoseconds))
