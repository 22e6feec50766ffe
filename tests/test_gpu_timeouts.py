"""Failure detection on the device: bounded waits report a timeout instead of hanging.

Every wait on an asynchronous copy or a tensor-core operation in the pipelined kernels is
bounded in wall-clock time.  With the limit set to 1 ns, the first wait that is not satisfied
at once gives up: the kernel stops, drains its own in-flight copies and MMAs, frees its tensor
memory and records WQ_ERR_TIMEOUT in the device status word.  Nothing traps or hangs, and the
context stays usable: after restoring the limit the same calls give the same results again.
"""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

WQ_ERR_TIMEOUT = 5


@pytest.fixture(scope="module")
def wq():
    import bit_gemv_gemm_group_b200 as m
    return m


def _cases(wq):
    g = np.random.default_rng(7)
    w = torch.from_numpy((g.standard_normal((4096, 4096)) * 0.02).astype(np.float16)).cuda()
    qw, sc, qz = wq.quantize_group_int4(w, 128)
    x1 = torch.from_numpy(workloads.activations(1, 4096, 0.01, 50.0, seed=7, tensor_id=1)).cuda()
    x64 = torch.from_numpy(workloads.activations(64, 4096, 0.01, 50.0, seed=7, tensor_id=2)).cuda()
    xq, sx = wq.quantize_int8_per_token(x64)
    w8, sw = wq.quantize_int8_per_channel(w)
    return {
        "streaming GEMV": lambda: wq.gemv_w4a16(x1, qw, sc, qz, 128),
        "tcgen05 W4A16 GEMM": lambda: wq.gemm_w4a16(x64, qw, sc, qz, 128),
        "tcgen05 W8A8 GEMM": lambda: wq.gemm_w8a8(xq, sx, w8, sw),
    }


def test_bounded_waits_time_out_and_the_context_recovers(wq):
    cases = _cases(wq)
    good = {}
    for name, fn in cases.items():
        good[name] = fn()
        assert wq.device_status() == 0, name
    try:
        for name, fn in cases.items():
            wq.set_wait_limit(1)
            fn()
            assert wq.device_status() == WQ_ERR_TIMEOUT, name
            wq.set_wait_limit(0)
            again = fn()  # the context is still usable and the kernel correct
            assert wq.device_status() == 0, name
            assert torch.equal(again.view(torch.int16), good[name].view(torch.int16)), name
    finally:
        wq.set_wait_limit(0)
        wq.device_status()
