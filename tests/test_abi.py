"""The C-ABI library loads, exports every entry point that include/wq.h declares, and
rejects bad arguments on the host (no GPU needed: validation runs before any CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wq.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wq_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def wq():
    import bit_gemv_gemm_group_b200 as m
    return m


def test_header_declares_the_hot_path():
    names = declared_functions()
    for required in ["wq_quantize_group_int4", "wq_quantize_int8_per_channel", "wq_quantize_int8_per_token",
                     "wq_smooth", "wq_gemv_w4a16", "wq_gemm_w4a16", "wq_gemm_w8a8", "wq_gemv_w8a16",
                     "wq_last_error", "wq_device_status"]:
        assert required in names


def test_library_exports_every_declared_symbol(wq):
    missing = [n for n in declared_functions() if not hasattr(wq.lib, n)]
    assert not missing, f"declared in wq.h but not exported: {missing}"


FAKE = ctypes.c_void_p(0x10000)       # aligned, never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10008)


def _err(wq):
    return wq.lib.wq_last_error().decode()


def test_null_and_alignment_rejected(wq):
    L = wq.lib
    assert L.wq_quantize_group_int4(None, 1, 4, 128, 128, FAKE, FAKE, FAKE, None) == wq.WQ_ERR_INVALID_ARG
    assert "w is null" in _err(wq)
    assert L.wq_quantize_group_int4(MISALIGNED, 1, 4, 128, 128, FAKE, FAKE, FAKE, None) == wq.WQ_ERR_ALIGNMENT
    assert L.wq_gemv_w4a16(FAKE, 1, FAKE, FAKE, FAKE, 16, 128, 128, None, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_gemm_w8a8(FAKE, FAKE, FAKE, FAKE, 16, 16, 16, MISALIGNED, None, None) == wq.WQ_ERR_ALIGNMENT


def test_sizes_rejected(wq):
    L = wq.lib
    # group size outside {32, 64, 128, 256}
    assert L.wq_quantize_group_int4(FAKE, 1, 4, 96, 96, FAKE, FAKE, FAKE, None) == wq.WQ_ERR_UNSUPPORTED
    # K not a multiple of the group
    assert L.wq_quantize_group_int4(FAKE, 1, 4, 192, 128, FAKE, FAKE, FAKE, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_quantize_group_int4(FAKE, 1, 0, 128, 128, FAKE, FAKE, FAKE, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_quantize_group_int4(FAKE, 7, 4, 128, 128, FAKE, FAKE, FAKE, None) == wq.WQ_ERR_INVALID_ARG
    # batch outside 1..8 for the GEMVs
    assert L.wq_gemv_w4a16(FAKE, 9, FAKE, FAKE, FAKE, 16, 128, 128, FAKE, None) == wq.WQ_ERR_UNSUPPORTED
    assert L.wq_gemv_w4a16(FAKE, 0, FAKE, FAKE, FAKE, 16, 128, 128, FAKE, None) == wq.WQ_ERR_UNSUPPORTED
    assert L.wq_gemv_w8a16(FAKE, 9, FAKE, FAKE, 16, 128, FAKE, None) == wq.WQ_ERR_UNSUPPORTED
    # W4A16 GEMM below 16 rows: only 9..15 rows with K % 256 == 0 (one streaming pass)
    assert L.wq_gemm_w4a16(FAKE, 12, FAKE, FAKE, FAKE, 16, 640, 128, FAKE, None) == wq.WQ_ERR_UNSUPPORTED
    assert L.wq_gemm_w4a16(FAKE, 8, FAKE, FAKE, FAKE, 16, 512, 128, FAKE, None) == wq.WQ_ERR_UNSUPPORTED
    assert "K % 256" in L.wq_last_error().decode()
    # K granularity of the INT8 paths
    assert L.wq_quantize_int8_per_token(FAKE, 4, 24, None, FAKE, FAKE, None) == wq.WQ_ERR_UNSUPPORTED
    assert L.wq_gemv_w8a16(FAKE, 1, FAKE, FAKE, 16, 24, FAKE, None) == wq.WQ_ERR_UNSUPPORTED
    assert L.wq_gemm_w8a8(FAKE, FAKE, FAKE, FAKE, 16, 16, 24, FAKE, None, None) == wq.WQ_ERR_UNSUPPORTED
    # W8A8: |acc| <= 128 * 128 * K must stay below 2^31; at K = 131072 (-128) * (-128) products
    # reach 2^31 exactly, so the largest K (a multiple of 16) is 131056
    assert L.wq_gemm_w8a8(FAKE, FAKE, FAKE, FAKE, 16, 16, 131072, FAKE, None, None) == wq.WQ_ERR_UNSUPPORTED
    assert "131056" in L.wq_last_error().decode()
    assert 128 * 128 * 131056 < 2 ** 31 <= 128 * 128 * 131072
    # both W4A16 matmuls take the group sizes the quantizer writes (32/64/128/256) and no other
    assert L.wq_gemm_w4a16(FAKE, 16, FAKE, FAKE, FAKE, 16, 512, 96, FAKE, None) == wq.WQ_ERR_UNSUPPORTED
    assert L.wq_gemv_w4a16(FAKE, 1, FAKE, FAKE, FAKE, 16, 512, 96, FAKE, None) == wq.WQ_ERR_UNSUPPORTED
    assert "32, 64, 128 or 256" in L.wq_last_error().decode()
    # smoothing: alpha range, K granularity
    assert L.wq_smooth(FAKE, 4, FAKE, 4, 64, ctypes.c_float(1.5), FAKE, FAKE, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_smooth(FAKE, 4, FAKE, 4, 60, ctypes.c_float(0.5), FAKE, FAKE, None) == wq.WQ_ERR_UNSUPPORTED


def test_workspace_size(wq):
    # column maxima of X and W (K padded to 4 words each) + one ticket per 256 columns (padded to 4)
    assert wq.smooth_workspace_bytes(8192) == (2 * 8192 + 32) * 4
    assert wq.smooth_workspace_bytes(10) == (2 * 12 + 4) * 4
    assert wq.smooth_workspace_bytes(1300) == (2 * 1300 + 8) * 4
    assert wq.smooth_workspace_bytes(0) == 0


def test_fp4_scale_bytes(wq):
    # 512-byte atoms: one per (128-row block, group of four factors); a factor per 32 (MXFP4) or 16 (NVFP4) values
    assert wq.fp4_scale_bytes(128, 256, False) == 1 * 2 * 512
    assert wq.fp4_scale_bytes(128, 256, True) == 1 * 4 * 512
    assert wq.fp4_scale_bytes(2048, 8192, True) == 16 * 128 * 512
    assert wq.fp4_scale_bytes(129, 160, False) == 2 * 2 * 512     # 5 factors -> 2 groups; 2 row blocks
    assert wq.fp4_scale_bytes(1, 16, True) == 512
    assert wq.fp4_scale_bytes(0, 256, True) == 0 and wq.fp4_scale_bytes(4, 0, False) == 0


def test_binding_rejects_cpu_tensors(wq):
    import torch
    with pytest.raises(ValueError, match="CUDA"):
        wq.quantize_group_int4(torch.zeros(4, 128, dtype=torch.float16))
