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


def _round_pair_rule(w, s):
    """The fp16 INT4 quantizer's division-free rounding: candidates from RN(1/s) one ulp down
    and one ulp up, the even one where they differ.  Returns (codes, any exact half-integer
    products); products are exact in fp64 (11-bit x 24-bit significands)."""
    rs = (np.float32(1.0) / np.float32(s)).astype(np.float32)
    bits = rs.view(np.uint32)
    rs_lo = (bits - np.uint32(1)).view(np.float32).astype(np.float64)
    rs_hi = (bits + np.uint32(1)).view(np.float32).astype(np.float64)
    x_lo, x_hi = w * rs_lo, w * rs_hi
    half = np.any(np.abs(x_lo - np.floor(x_lo)) == 0.5) or np.any(np.abs(x_hi - np.floor(x_hi)) == 0.5)
    n_lo, n_hi = np.rint(x_lo), np.rint(x_hi)
    pick_hi = (n_lo != n_hi) & (np.mod(n_lo, 2) != 0)
    return np.where(pick_hi, n_hi, n_lo), half, n_lo, n_hi


def _mean_rule(n_lo, n_hi):
    """The kernel's tie-break on the fp32 pipe: the candidates as M + n (M = 1.5 * 2^23), the
    exact half of one plus the other times 1/2 rounded once (a fused multiply-add), minus M.
    The fp64 sum is exact (integers and halves near 2^23), so one conversion to fp32 is the
    fused rounding."""
    M = np.float64(1.5 * 2.0 ** 23)
    rl = (M + n_lo).astype(np.float32)
    half_rh = ((M + n_hi).astype(np.float32) * np.float32(0.5)).astype(np.float32)
    assert np.array_equal(half_rh.astype(np.float64) * 2, M + n_hi)  # the halving is exact
    mean = (rl.astype(np.float64) * 0.5 + half_rh.astype(np.float64)).astype(np.float32)
    return mean.astype(np.float64) - M


def test_int4_division_free_rounding_is_exact():
    # For fp16 weights w and fp16 scales s with |w / s| < 32 the rule must give rne(fl32(w / s))
    # for every w, and no fused sum may land exactly on a half-integer (where the hardware's
    # own tie-break would decide).  All finite fp16 w; every power-of-two s and 3000 others.
    hw = np.arange(0x10000, dtype=np.uint32).astype(np.uint16)
    w16 = hw.view(np.float16)
    w16 = w16[np.isfinite(w16)]
    w = w16.astype(np.float64)
    g = np.random.default_rng(11)
    pos = np.arange(1, 0x7C00, dtype=np.uint16)
    pow2 = pos[(pos & 0x3FF) == 0]
    sub_pow2 = np.array([1 << i for i in range(10)], np.uint16)
    pick = np.concatenate([pow2, sub_pow2, g.choice(pos, 3000, replace=False)])
    for sb in pick:
        s = np.float64(np.array([sb], np.uint16).view(np.float16)[0])
        ww = w[np.abs(w / s) < 32]
        got, half, n_lo, n_hi = _round_pair_rule(ww, s)
        ref = np.rint((ww.astype(np.float32) / np.float32(s)).astype(np.float64))
        assert not half, sb
        assert np.array_equal(got, ref), (sb, ww[got != ref][:4])
        # the candidates differ by at most one, and the rounded mean picks the same code
        assert np.all(np.abs(n_lo - n_hi) <= 1), sb
        assert np.array_equal(_mean_rule(n_lo, n_hi), got), sb


def test_div6_by_fp64_product_is_correctly_rounded():
    # The NVFP4 quantizer takes a block's max |v| / 6 as the fp64 product with RN64(1/6) rounded to
    # fp32.  The dividend is an fp16 value, so every case is checked: all finite non-negative fp16.
    inv6 = np.float64(1.0) / np.float64(6.0)
    assert inv6.view(np.uint64) == 0x3FC5555555555555
    h = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16)
    a32 = h.astype(np.float32)
    ieee = a32 / np.float32(6.0)
    fast = (a32.astype(np.float64) * inv6).astype(np.float32)
    assert np.array_equal(ieee.view(np.uint32), fast.view(np.uint32))
