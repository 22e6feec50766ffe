"""CPU checks of arithmetic shortcuts the CUDA kernels rely on (no GPU, no oracle).

The INT4 quantizer computes the fp32 quotient (hi - lo) / 15 as the fp64 product
(hi - lo) * RN64(1/15) rounded to fp32.  The claim is that this equals the IEEE fp32
quotient for every fp32 dividend; the argument only depends on the dividend's 24-bit
significand, so checking every significand (and a few scalings) covers all inputs.
"""
import numpy as np


def test_div15_by_fp64_product_is_correctly_rounded():
    inv15 = np.float64(1.0) / np.float64(15.0)
    assert inv15.view(np.uint64) == 0x3FB1111111111111
    m = np.arange(1 << 23, 1 << 24, dtype=np.float64)
    for e in (-40, -24, 0, 7):
        d32 = (m * 2.0 ** e).astype(np.float32)
        assert np.array_equal(d32.astype(np.float64), m * 2.0 ** e)  # exact fp32 dividends
        ieee = d32 / np.float32(15.0)
        fast = (d32.astype(np.float64) * inv15).astype(np.float32)
        assert np.array_equal(ieee.view(np.uint32), fast.view(np.uint32)), e
    # small significands and zero
    d32 = np.arange(0, 1 << 12, dtype=np.float32)
    assert np.array_equal((d32 / np.float32(15.0)).view(np.uint32),
                          (d32.astype(np.float64) * inv15).astype(np.float32).view(np.uint32))
