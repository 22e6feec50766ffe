"""Failure detection on the device: bounded waits report a timeout instead of hanging.

Every wait on an asynchronous copy or a tensor-core operation in the pipelined kernels is
bounded in wall-clock time.  A wait that runs out records WQ_ERR_TIMEOUT in the device status
word; the kernel stops, drains its own in-flight copies and MMAs and frees its tensor memory.
A self-test kernel waits on a barrier that nothing completes, so its timeout is certain; the
pipelined kernels run under a 1 ns limit, where they finish or stop early.  Nothing traps or
hangs, and the context stays usable: with the limit restored the same calls give the same
results again.
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
        "bulk-copy ring INT4 quantizer": lambda: wq.quantize_group_int4(w, 128)[0].view(torch.int16),
    }


def test_a_wait_that_nothing_completes_times_out(wq):
    wq.set_wait_limit(1_000_000)  # 1 ms
    try:
        wq.selftest_wait_timeout()
        assert wq.device_status() == WQ_ERR_TIMEOUT
        assert wq.device_status() == 0  # reading the word clears it
    finally:
        wq.set_wait_limit(0)


def test_pipelined_kernels_give_up_cleanly_and_the_context_recovers(wq):
    # With a 1 ns limit a kernel either finishes (every wait was satisfied before the
    # timer advanced) or stops early through its abort path; either way nothing hangs,
    # and with the limit restored the same calls give the same bits.
    cases = _cases(wq)
    good = {}
    for name, fn in cases.items():
        good[name] = fn()
        assert wq.device_status() == 0, name
    try:
        for name, fn in cases.items():
            wq.set_wait_limit(1)
            fn()
            assert wq.device_status() in (0, WQ_ERR_TIMEOUT), name
            wq.set_wait_limit(0)
            again = fn()
            assert wq.device_status() == 0, name
            assert torch.equal(again.view(torch.int16), good[name].view(torch.int16)), name
    finally:
        wq.set_wait_limit(0)
        wq.device_status()
