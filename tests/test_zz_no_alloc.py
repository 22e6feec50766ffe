"""wq_smooth_noalloc: SmoothQuant factors for callers that cannot allocate device memory.

Such callers (a plug-in inside an engine that owns all device memory, or a path that may not
call cudaMalloc) get the workspace from a fixed array that the library keeps on the device.
These tests call the entry point through the C ABI and compare it with wq_smooth, which uses a
caller-owned workspace.  The file is named so that pytest collects it last.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle

FAKE = ctypes.c_void_p(0x10000)  # aligned and never dereferenced: validation fails first
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "wq.h")


def header_max_k():
    """The limit as the C header states it (the value the library was compiled with)."""
    m = re.search(r"#define\s+WQ_SMOOTH_NOALLOC_MAX_K\s+(\d+)", open(HEADER).read())
    assert m, "WQ_SMOOTH_NOALLOC_MAX_K not found in include/wq.h"
    return int(m.group(1))


@pytest.fixture(scope="module")
def wq():
    import bit_gemv_gemm_group_b200 as m
    return m


def test_noalloc_rejects_k_beyond_the_builtin_workspace(wq):
    # Host-side check before any CUDA call: runs without a GPU.  The limit comes from the header;
    # the output pointer is null, so even a library built with a larger limit would stop at
    # argument validation and never launch on the fake addresses.
    limit = header_max_k()
    assert wq.SMOOTH_NOALLOC_MAX_K == limit
    st = wq.lib.wq_smooth_noalloc(FAKE, 4, FAKE, 4, limit + 8, ctypes.c_float(0.5), None, None)
    assert st == wq.WQ_ERR_UNSUPPORTED
    assert "exceeds the built-in workspace" in wq.lib.wq_last_error().decode()


def _inputs(M, N, K, seed, outlier):
    g = np.random.default_rng(seed)
    X = g.standard_normal((M, K)).astype(np.float32)
    X[:, g.choice(K, size=max(1, K // 50), replace=False)] *= outlier
    X[:, 0] = 0.0  # an all-zero column hits the 1e-5 clamp
    W = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    return (torch.from_numpy(X.astype(np.float16)).cuda(), torch.from_numpy(W.astype(np.float16)).cuda())


def _noalloc_via_abi(wq, X, W, alpha):
    M, K = X.shape
    N = W.shape[0]
    s = torch.empty(K, dtype=torch.float32, device=X.device)
    st = wq.lib.wq_smooth_noalloc(ctypes.c_void_p(X.data_ptr()), M, ctypes.c_void_p(W.data_ptr()), N, K,
                                  ctypes.c_float(alpha), ctypes.c_void_p(s.data_ptr()),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == wq.WQ_OK, wq.lib.wq_last_error().decode()
    return s


@pytest.mark.gpu
def test_noalloc_matches_wq_smooth_on_two_calls_in_a_row(wq):
    # The first call leaves large column maxima over a wide K in the shared array; the second
    # (smaller K, smaller values) must not see them.  Smoothing factors are compared bit for bit,
    # as in the other smoothing tests (alpha = 0.5 is correctly rounded on both paths).
    cases = [((300, 257, 4096, 11, 200.0), 0.5), ((37, 90, 1032, 12, 3.0), 0.5)]
    for (M, N, K, seed, outlier), alpha in cases:
        X, W = _inputs(M, N, K, seed, outlier)
        got = _noalloc_via_abi(wq, X, W, alpha)
        want = wq.smooth(X, W, alpha)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int32), want.view(torch.int32)), f"M={M} N={N} K={K}"
    wq.device_status()


@pytest.mark.gpu
def test_noalloc_at_the_maximum_k(wq):
    # The whole built-in array in use, against wq_smooth and against the CPU oracle (few rows, so
    # the oracle stays fast): bit for bit at alpha = 0.5, within 1 ulp at 0.75 (fp64 pow rounded
    # to fp32 on both sides, as in the other smoothing tests).
    K = header_max_k()
    X, W = _inputs(3, 5, K, 13, 60.0)
    Xh, Wh = X.cpu().numpy(), W.cpu().numpy()
    for alpha in (0.5, 0.75):
        got = _noalloc_via_abi(wq, X, W, alpha)
        want = wq.smooth(X, W, alpha)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int32), want.view(torch.int32)), f"alpha={alpha}"
        ref = oracle.smooth_factors(Xh, Wh, alpha)
        ulps = np.abs(got.cpu().numpy().view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
        assert ulps.max() <= (0 if alpha == 0.5 else 1), f"alpha={alpha}: {ulps.max()} ulp from the oracle"
