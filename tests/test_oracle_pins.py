"""Pins for the CPU oracle: page-printed values, closed forms, invariants, special
cases that reduce to library routines, and brute force on tiny inputs.

Each check is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a wrong rounding mode) fails one of
them.  These run without a GPU.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# binary16 conversion against numpy's independent implementation
# --------------------------------------------------------------------------
def test_half_to_float_all_bit_patterns():
    L = oracle.lib()
    bits = np.arange(65536, dtype=np.uint32)
    ours = np.array([L.orc_half_to_float(int(b)) for b in bits], np.float32)
    ref = bits.astype(np.uint16).view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_float_to_half_matches_numpy_rne():
    L = oracle.lib()
    g = np.random.default_rng(1)
    # random bit patterns over the whole fp16-relevant exponent range, plus edges
    mant = g.integers(0, 1 << 23, 40000, dtype=np.uint32)
    expo = g.integers(127 - 27, 127 + 17, 40000, dtype=np.uint32)
    sign = g.integers(0, 2, 40000, dtype=np.uint32)
    f = ((sign << 31) | (expo << 23) | mant).view(np.float32)
    edges = np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 70000.0, 2 ** -24, 2 ** -25,
                      3 * 2 ** -25, 2 ** -14, 2 ** -14 - 2 ** -25, 1.0 + 2 ** -11,
                      1.0 + 3 * 2 ** -11, 0.1, 0.128, 0.052, 1e-8, -2 ** -26], np.float32)
    f = np.concatenate([f, edges, -edges])
    with np.errstate(over="ignore"):
        ref = f.astype(np.float16).view(np.uint16)
    ours = np.array([L.orc_float_to_half(float(v)) for v in f], np.uint16)
    assert np.array_equal(ours, ref)


# --------------------------------------------------------------------------
# INT4 asymmetric: the pages' worked examples
# --------------------------------------------------------------------------
def test_int4_six_weight_worked_example():
    d = gold("int4_worked_six_weights.json")
    w = np.zeros((1, d["pad_with_zeros_to"]), np.float32)
    w[0, :6] = d["weights"]
    qw, sc, qz = oracle.quantize_group_int4(w, group_size=8)
    codes = oracle.unpack_int4_codes(qw, 8)[0]
    z = oracle.unpack_int4_zeros(qz, 1)[0, 0]
    s = float(sc[0, 0])
    assert round(s, 3) == d["scale"]
    assert z == d["zero_point"]
    assert list(codes[:6]) == d["codes"]
    assert list(codes[6:]) == [z, z]                  # the exact zeros land on z
    back = oracle.dequant_int4(qw, sc, qz, 8, 8)[0, :6]
    assert [round(v, 3) for v in back] == d["dequantized_3dp"]
    err = np.abs(back - np.asarray(d["weights"]))
    assert round(err.max(), 3) == d["max_abs_error"]
    assert err.max() <= s / 2 and round(s / 2, 3) == d["half_step"]


def test_int4_eight_weight_worked_example():
    d = gold("int4_worked_eight_weights.json")
    w = np.asarray([d["weights"]], np.float32)
    qw, sc, qz = oracle.quantize_group_int4(w, group_size=8)
    assert round(float(sc[0, 0]), 4) == d["scale_4dp"]
    assert oracle.unpack_int4_zeros(qz, 1)[0, 0] == d["zero_point"]
    assert list(oracle.unpack_int4_codes(qw, 8)[0]) == d["codes"]
    back = oracle.dequant_int4(qw, sc, qz, 8, 8)[0]
    assert [round(v, 3) + 0.0 for v in back] == d["dequantized_3dp"]


def test_int4_fp16_input_path_matches_fp32_path():
    # The same values given as fp16 and as the fp32 of those fp16 values quantize identically.
    g = np.random.default_rng(2)
    w16 = (g.standard_normal((8, 256)) * 0.02).astype(np.float16)
    a = oracle.quantize_group_int4(w16, 128)
    b = oracle.quantize_group_int4(w16.astype(np.float32), 128)
    for x, y in zip(a, b):
        assert np.array_equal(np.asarray(x).view(np.uint8), np.asarray(y).view(np.uint8))


# --------------------------------------------------------------------------
# INT4 invariants: error bound s/2, exact zero, range coverage, packing layout
# --------------------------------------------------------------------------
def _int4_case(seed=3, N=64, K=1024, g=128):
    r = np.random.default_rng(seed)
    w = (r.standard_normal((N, K)) * 0.02).astype(np.float32)
    w.reshape(-1)[96::97] *= 20                        # outliers, as in the tiny workload
    w[:, 5::37] = 0.0                                  # exact zeros
    w[3, :128] = 0.0                                   # an all-zero group
    w[4, 128:256] = 0.25                               # a constant group
    w[5, 256:384] = np.abs(w[5, 256:384]) + 0.01       # an all-positive group
    w[6, 384:512] = -np.abs(w[6, 384:512]) - 0.01      # an all-negative group
    return w, oracle.quantize_group_int4(w, g)


def test_int4_error_bound_half_step():
    w, (qw, sc, qz) = _int4_case()
    N, K = w.shape
    s = np.repeat(sc.astype(np.float64), 128, axis=1)
    z = np.repeat(oracle.unpack_int4_zeros(qz, K // 128), 128, axis=1)
    back = oracle.dequant_int4(qw, sc, qz, K)
    pre = np.rint(w / s) + z                           # pre-clamp code (float reading)
    inside = (pre >= 0) & (pre <= 15)
    err = np.abs(back - w)
    slack = np.spacing(np.abs(w).astype(np.float32)).astype(np.float64) + 2 ** -40
    assert np.all(err[inside] <= s[inside] / 2 + slack[inside] + s[inside] * 2 ** -22)
    # with the range widened to contain 0 and the fp16 scale, clipping is at most one step
    assert np.all(err <= 1.5 * s)


def test_int4_zero_maps_exactly():
    w, (qw, sc, qz) = _int4_case()
    back = oracle.dequant_int4(qw, sc, qz, w.shape[1])
    assert np.all(back[w == 0.0] == 0.0)
    assert np.all(back[3, :128] == 0.0) and sc[3, 0] == np.float16(1.0)


def test_int4_constant_and_one_signed_groups():
    w, (qw, sc, qz) = _int4_case()
    K = w.shape[1]
    z = oracle.unpack_int4_zeros(qz, K // 128)
    codes = oracle.unpack_int4_codes(qw, K)
    # constant 0.25: range [0, 0.25] -> s = fp16(0.25/15), z = 0, codes 15
    assert sc[4, 1] == np.float16(np.float32(0.25) / np.float32(15))
    assert z[4, 1] == 0 and np.all(codes[4, 128:256] == 15)
    # all-positive group: z = 0, the maximum gets code 15; all-negative: z = 15
    assert z[5, 2] == 0 and codes[5, 256:384].max() == 15
    assert z[6, 3] == 15 and codes[6, 384:512].min() == 0


def test_int4_packing_order_nibbles():
    # values (c - 7) * 0.125 for c = 0..15 give s = 0.125 exactly, z = 7 and codes c; read back
    # through the documented layout: element k -> nibble (k mod 8) of word k // 8.
    K = 1024
    base = (np.arange(16, dtype=np.float32) - 7) * np.float32(0.125)
    w = np.tile(base, K // 16)[None, :].copy()
    qw, sc, qz = oracle.quantize_group_int4(w, 128)
    codes = oracle.unpack_int4_codes(qw, K)[0]
    assert np.array_equal(codes, np.tile(np.arange(16), K // 16))
    word0 = int(qw[0, 0])
    assert [(word0 >> (4 * i)) & 0xF for i in range(8)] == list(range(8))
    assert qz.shape == (1, 1) and int(qz[0, 0]) == 0x77777777 and np.all(sc == np.float16(0.125))


def test_storage_overhead_and_70b_estimate():
    d = gold("storage_overhead.json")
    N, K, g = 256, 8192, d["group"]
    w = np.zeros((N, K), np.float16)
    qw, sc, qz = oracle.quantize_group_int4(w, g)
    bits_per_weight_overhead = 8 * (sc.nbytes + qz.nbytes) / (N * K)
    assert bits_per_weight_overhead == d["overhead_bits_per_weight"]
    bytes_per_param = (qw.nbytes + sc.nbytes + qz.nbytes) / (N * K)
    assert bytes_per_param == d["bytes_per_param"]
    assert round(d["params"] * bytes_per_param / 1e9, 1) == d["total_gb_1dp"]


# --------------------------------------------------------------------------
# Symmetric quantization: the pages' INT8 and INT4 examples
# --------------------------------------------------------------------------
def test_int8_worked_example_with_outlier():
    d = gold("int8_worked_outlier.json")
    w = np.asarray([d["weights"]], np.float16)
    q, s = oracle.quantize_int8_per_channel(w)
    assert q[0, 1] == d["code_of_0.12"]
    back = q.astype(np.float64) * s[0]
    assert np.all(np.abs(back - w.astype(np.float64)) <= s[0] / 2 + 1e-12)   # half a step
    w2 = np.asarray([d["weights"] + [d["outlier"]]], np.float16)
    q2, s2 = oracle.quantize_int8_per_channel(w2)
    assert round(float(s2[0] / s[0]), 1) == d["step_ratio_with_outlier"]
    assert q2[0, 0] == d["code_of_0.04_with_outlier"]
    lost = 1 - q2[0, 1] * float(s2[0]) / float(w2[0, 1])
    assert round(100 * lost) == d["loss_of_0.12_with_outlier_percent"]


def test_symmetric_int4_exercises():
    d = gold("symmetric_int4_exercises.json")
    e = d["exercise_step"]
    q, s = oracle.quantize_sym_rows(np.asarray([e["group"]], np.float16), bits=4)
    assert round(float(s[0]), 4) == e["scale_4dp"] and q[0, 1] == e["code_of_0.05"]
    o = d["outlier_group"]
    q, s = oracle.quantize_sym_rows(np.asarray([o["group"]], np.float16), bits=4)
    assert round(float(s[0]), 2) == o["scale_2dp"]
    small = [i for i, v in enumerate(o["group"]) if abs(v) < 1]
    assert np.all(q[0, small] == o["small_codes"]) and q[0, 4] == 7


def test_int8_codes_range_and_bound():
    g = np.random.default_rng(4)
    x = (g.standard_normal((32, 512)) * 3).astype(np.float16)
    x[:, 7] *= 50
    x[5] = 0                                            # all-zero row: scale clamp 1e-8/127
    q, s = oracle.quantize_int8_per_token(x)
    assert s[5] == np.float32(1e-8) / np.float32(127) and np.all(q[5] == 0)
    assert q.min() >= -127 and q.max() <= 127           # absmax row scale never needs -128
    assert np.all(np.abs(q).max(axis=1)[np.arange(32) != 5] == 127)
    back = q.astype(np.float64) * s[:, None].astype(np.float64)
    err = np.abs(back - x.astype(np.float64))
    assert np.all(err <= s[:, None] / 2 * (1 + 2 ** -20) + 1e-30)


def test_int8_smoothing_direction():
    # mode 1 multiplies by s_j, mode 2 divides: x = s (exactly representable) -> x/s = 1, w*s = s^2
    s = np.asarray([2.0, 4.0, 0.5, 8.0], np.float32)
    x = np.asarray([[2.0, 4.0, 0.5, 8.0]], np.float16)
    qx, sx = oracle.quantize_int8_per_token(x, s)
    assert np.all(qx == 127)                            # x / s == 1 everywhere
    qw, sw = oracle.quantize_int8_per_channel(x, s)
    assert sw[0] == np.float32(64.0) / np.float32(127)  # max of w*s is 8*8
    assert qw[0, 3] == 127 and qw[0, 2] == round(0.25 / (64 / 127))


# --------------------------------------------------------------------------
# SmoothQuant factors
# --------------------------------------------------------------------------
def test_smooth_closed_forms():
    X = np.zeros((3, 5), np.float16)
    W = np.zeros((4, 5), np.float16)
    X[1, 0], W[2, 0] = -4.0, 1.0        # sqrt(4)/sqrt(1) = 2
    X[0, 1], W[3, 1] = 9.0, -0.25       # 3 / 0.5 = 6
    X[2, 2], W[0, 2] = 0.25, 16.0       # 0.5 / 4 = 0.125
    W[1, 3] = 4.0                       # X column all zero -> clamp 1e-5
    # column 4 all zero in both -> 1
    s = oracle.smooth_factors(X, W, 0.5)
    assert s[0] == 2.0 and s[1] == 6.0 and s[2] == 0.125
    assert s[3] == np.float32(np.sqrt(np.float32(1e-5))) / np.float32(2.0)
    assert s[4] == 1.0
    # alpha = 1: s = max|X_j| ; alpha = 0: s = 1 / max|W_j|
    s1 = oracle.smooth_factors(X, W, 1.0)
    assert s1[0] == 4.0 and s1[1] == 9.0 and s1[2] == 0.25
    s0 = oracle.smooth_factors(X, W, 0.0)
    assert s0[0] == 1.0 and s0[1] == 4.0 and s0[2] == np.float32(1 / 16)


def test_smooth_balances_columns_and_orientation():
    # alpha = 0.5 equalizes max|X_j / s_j| and max|W_j * s_j| (= sqrt(ax*aw)); non-square
    # shapes catch a max taken over the wrong axis of W [out, in].
    g = np.random.default_rng(5)
    X = g.standard_normal((48, 96)).astype(np.float16)
    X[:, [3, 17, 60]] *= 40
    W = (g.standard_normal((80, 96)) * 0.05).astype(np.float16)
    s = oracle.smooth_factors(X, W, 0.5).astype(np.float64)
    mx = np.abs(X.astype(np.float64) / s).max(axis=0)
    mw = np.abs(W.astype(np.float64) * s).max(axis=0)
    assert np.allclose(mx, mw, rtol=1e-6)
    # and the factor tracks the activation outliers
    assert np.all(s[[3, 17, 60]] > 4 * np.median(s))


def test_smoothquant_equivalence_exact_in_fp64():
    # (X diag(s)^-1)(diag(s) W)^T = X W^T  ("How quantization works", SmoothQuant; the
    # engine-room chapter's Y = (X diag(s)^-1)(diag(s) W))
    g = np.random.default_rng(6)
    X = g.standard_normal((16, 64)).astype(np.float16)
    W = (g.standard_normal((24, 64)) * 0.02).astype(np.float16)
    s = oracle.smooth_factors(X, W, 0.5).astype(np.float64)
    Y = X.astype(np.float64) @ W.astype(np.float64).T
    Ys = (X.astype(np.float64) / s) @ (W.astype(np.float64) * s).T
    assert np.max(np.abs(Ys - Y)) <= 1e-12 * np.max(np.abs(Y))


# --------------------------------------------------------------------------
# matmul references: special cases that reduce to library routines / closed forms
# --------------------------------------------------------------------------
def test_w4a16_ref_reduces_to_dequant_and_numpy_matmul():
    w, (qw, sc, qz) = _int4_case(seed=7, N=24, K=256)
    K = 256
    what = oracle.dequant_int4(qw, sc, qz, K)
    g = np.random.default_rng(8)
    x = g.standard_normal((3, K)).astype(np.float16)
    y, bound = oracle.matmul_w4a16_ref(x, qw, sc, qz, K)
    ref = x.astype(np.float64) @ what.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-15)
    assert np.allclose(bound, np.abs(x.astype(np.float64)) @ np.abs(what).T, rtol=1e-12)
    # one-hot activations pick out single dequantized weights (catches a transposed operand)
    e = np.zeros((2, K), np.float16)
    e[0, 17], e[1, 200] = 1.0, 1.0
    y1, _ = oracle.matmul_w4a16_ref(e, qw, sc, qz, K)
    assert np.array_equal(y1[0], what[:, 17]) and np.array_equal(y1[1], what[:, 200])
    # selected rows agree with the full result
    ys, _ = oracle.matmul_w4a16_ref(x, qw, sc, qz, K, rows=[5, 0, 23])
    assert np.array_equal(ys, y[:, [5, 0, 23]])


def test_w8a8_ref_is_exact_integer_matmul():
    g = np.random.default_rng(9)
    xq = g.integers(-128, 128, (7, 48), dtype=np.int8)
    wq = g.integers(-128, 128, (9, 48), dtype=np.int8)
    sx = g.random(7, dtype=np.float32) + 0.5
    sw = g.random(9, dtype=np.float32) + 0.5
    acc, y, bound = oracle.gemm_w8a8_ref(xq, sx, wq, sw)
    ref = xq.astype(np.int64) @ wq.astype(np.int64).T
    assert np.array_equal(acc, ref)
    assert np.allclose(y, ref * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64),
                       rtol=1e-15)
    # every pair of int8 codes (K = 1): the products themselves
    a = np.arange(-128, 128, dtype=np.int8)[:, None]
    acc1, _, _ = oracle.gemm_w8a8_ref(a, np.ones(256, np.float32), a, np.ones(256, np.float32))
    assert np.array_equal(acc1, np.outer(np.arange(-128, 128), np.arange(-128, 128)))
    # the worst case for K = 8192 stays inside int32 (|acc| <= 128^2 * 8192 = 2^27)
    big = np.full((1, 8192), -128, np.int8)
    acc2, _, _ = oracle.gemm_w8a8_ref(big, np.ones(1, np.float32), big, np.ones(1, np.float32))
    assert acc2[0, 0] == 128 * 128 * 8192
    # selected rows of X (ms) and of W (ns), in any order and with repeats, agree with the
    # full result indexed the same way (a swapped or misapplied selection fails here)
    ms, ns = [6, 0, 3, 3], [8, 1, 4]
    accs, ys, bs = oracle.gemm_w8a8_ref(xq, sx, wq, sw, ms=ms, ns=ns)
    assert np.array_equal(accs, acc[np.ix_(ms, ns)])
    assert np.array_equal(ys, y[np.ix_(ms, ns)]) and np.array_equal(bs, bound[np.ix_(ms, ns)])
    acc_m, _, _ = oracle.gemm_w8a8_ref(xq, sx, wq, sw, ms=[2])
    acc_n, _, _ = oracle.gemm_w8a8_ref(xq, sx, wq, sw, ns=[7, 5])
    assert np.array_equal(acc_m, acc[[2]]) and np.array_equal(acc_n, acc[:, [7, 5]])


def test_w8a16_ref_reduces_to_numpy():
    g = np.random.default_rng(10)
    wq = g.integers(-127, 128, (12, 96), dtype=np.int8)
    sw = (g.random(12, dtype=np.float32) + 0.1) * 0.01
    x = g.standard_normal((2, 96)).astype(np.float16)
    y, b = oracle.matmul_w8a16_ref(x, wq, sw)
    what = wq.astype(np.float64) * sw[:, None].astype(np.float64)
    assert np.allclose(y, x.astype(np.float64) @ what.T, rtol=1e-12, atol=1e-15)
    assert np.allclose(b, np.abs(x.astype(np.float64)) @ np.abs(what).T, rtol=1e-12)
    # selected rows (any order) agree with the full result's columns
    ys, bs = oracle.matmul_w8a16_ref(x, wq, sw, rows=[11, 0, 4])
    assert np.array_equal(ys, y[:, [11, 0, 4]]) and np.array_equal(bs, b[:, [11, 0, 4]])


# --------------------------------------------------------------------------
# direction-only statistics the pages assert (finer granularity -> less error,
# SmoothQuant between weight-only and plain W8A8)
# --------------------------------------------------------------------------
def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def test_granularity_orderings():
    g = np.random.default_rng(11)
    W = (g.standard_normal((64, 1024)) * np.exp(g.normal(np.log(0.02), 0.5, (64, 1)))).astype(np.float16)
    W.reshape(-1)[g.random(W.size) < 0.001] *= 30
    Wd = W.astype(np.float64)
    q, s = oracle.quantize_sym_rows(W.reshape(1, -1), bits=8)          # per tensor
    e_t = _rel((q.astype(np.float64) * s[0]).reshape(W.shape), Wd)
    q, s = oracle.quantize_int8_per_channel(W)                          # per channel
    e_c = _rel(q.astype(np.float64) * s[:, None], Wd)
    assert e_c < e_t
    qw, sc, qz = oracle.quantize_group_int4(W, 1024)                   # INT4 per channel
    e4c = _rel(oracle.dequant_int4(qw, sc, qz, 1024, 1024), Wd)
    qw, sc, qz = oracle.quantize_group_int4(W, 128)                    # INT4 per group
    e4g = _rel(oracle.dequant_int4(qw, sc, qz, 1024, 128), Wd)
    assert e4g < e4c and e_c < e4g


def test_smoothquant_error_ordering():
    g = np.random.default_rng(12)
    X = g.standard_normal((128, 256)).astype(np.float32)
    X[:, [4, 77, 150, 201]] *= 40
    X = X.astype(np.float16)
    W = (g.standard_normal((192, 256)) * 0.02).astype(np.float16)
    Xd, Wd = X.astype(np.float64), W.astype(np.float64)
    Y = Xd @ Wd.T
    qw, sw = oracle.quantize_int8_per_channel(W)
    Wq = qw * sw[:, None].astype(np.float64)
    err_w8 = _rel(Xd @ Wq.T, Y)
    qx, sx = oracle.quantize_sym_rows(X.reshape(1, -1), bits=8)        # per-tensor X as on the page
    Xq = (qx.astype(np.float64) * sx[0]).reshape(X.shape)
    err_w8a8 = _rel(Xq @ Wq.T, Y)
    s = oracle.smooth_factors(X, W, 0.5)
    qws, sws = oracle.quantize_int8_per_channel(W, s)
    Xs = (X.astype(np.float32) / s).astype(np.float32)
    qxs = np.rint(Xs / (np.abs(Xs).max() / np.float32(127)))           # per tensor, for the ordering
    Xsq = qxs.astype(np.float64) * float(np.abs(Xs).max() / np.float32(127))
    err_sq = _rel(Xsq @ (qws * sws[:, None].astype(np.float64)).T, Y)
    assert err_w8 < err_sq < err_w8a8
    # per-token on the smoothed activations (the path's granularity) is better still
    qxt, sxt = oracle.quantize_int8_per_token(X, s)
    err_sq_tok = _rel((qxt * sxt[:, None].astype(np.float64)) @ (qws * sws[:, None].astype(np.float64)).T, Y)
    assert err_sq_tok < err_w8a8


def test_bad_arguments_rejected():
    with pytest.raises(ValueError):
        oracle.quantize_group_int4(np.zeros((2, 100), np.float16), 128)
    with pytest.raises(ValueError):
        oracle.quantize_sym_rows(np.zeros((2, 8), np.float16), bits=9)


# --------------------------------------------------------------------------
# FP8 E4M3: the format pinned to torch's float8_e4m3fn conversions (an
# independent library implementation), the pages' 448 maximum and scale
# rule, and closed-form error bounds
# --------------------------------------------------------------------------
def _torch_e4m3_decode(codes):
    import torch
    return torch.tensor(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).float().numpy()


def test_e4m3_decode_all_codes_matches_torch_and_pages():
    codes = np.arange(256)
    ours = np.array([oracle.e4m3_to_float(c) for c in codes], np.float32)
    ref = _torch_e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and list(codes[nan]) == [0x7F, 0xFF]
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    # "E4M3 ... reaches +-448" (the largest finite code); no infinities
    assert np.nanmax(ours) == 448.0 and np.nanmin(ours) == -448.0 and not np.isinf(ours).any()
    assert oracle.e4m3_to_float(0x01) == 2.0 ** -9       # smallest subnormal
    assert oracle.e4m3_to_float(0x08) == 2.0 ** -6       # smallest normal


def test_e4m3_encode_matches_torch_rne():
    import torch
    g = np.random.default_rng(21)
    # every finite code, every midpoint between neighbours (ties to even), and random values
    fin = np.array([oracle.e4m3_to_float(c) for c in range(0x7F)], np.float64)   # 0 .. 448
    mids = (fin[:-1] + fin[1:]) / 2
    rnd = np.exp(g.uniform(np.log(2.0 ** -12), np.log(448.0), 20000))
    vals = np.concatenate([fin, mids, rnd, mids * (1 + 2 ** -20), mids * (1 - 2 ** -20)])
    vals = np.concatenate([vals, -vals]).astype(np.float32)
    ours = np.array([oracle.float_to_e4m3(v) for v in vals], np.uint8)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    # ties to even: 17 lies halfway between 16 (mantissa 0) and 18 (mantissa 1) -> 16
    assert oracle.e4m3_to_float(oracle.float_to_e4m3(17.0)) == 16.0
    assert oracle.e4m3_to_float(oracle.float_to_e4m3(19.0)) == 20.0
    # beyond the largest finite value the reading saturates to 448 (the format has no infinity)
    for v in (448.0, 460.0, 470.0, 1e6):
        assert oracle.float_to_e4m3(v) == 0x7E and oracle.float_to_e4m3(-v) == 0xFE


def test_fp8_quantizer_scale_rule_and_error_bound():
    # "scale = max|w| / 448": the largest magnitude maps to the largest code, exactly
    g = np.random.default_rng(22)
    w = (g.standard_normal((6, 256)) * 0.02).astype(np.float32)
    w.reshape(-1)[96::97] *= 20
    w = w.astype(np.float16)
    for per_row in (True, False):
        q, s = oracle.quantize_fp8_e4m3(w, per_row=per_row)
        wf = w.astype(np.float32)
        amax = np.abs(wf).max(axis=1) if per_row else np.full(6, np.abs(wf).max())
        assert np.array_equal(s, (amax / np.float32(448.0)).astype(np.float32)[: s.size])
        dec = _torch_e4m3_decode(q).astype(np.float64)
        srow = (s if per_row else np.repeat(s, 6)).astype(np.float64)[:, None]
        what = dec * srow
        # relative error at most half a step of a 3-bit mantissa (2^-4) on the normal range,
        # absolute error at most half the subnormal step (2^-10 * s) below it
        v = wf.astype(np.float64) / srow
        err = np.abs(what - wf)
        lim = np.where(np.abs(v) >= 2.0 ** -6, 2.0 ** -4 * np.abs(wf), 2.0 ** -10 * srow) * (1 + 1e-6)
        assert np.all(err <= lim)
        for r in range(6):
            k = np.argmax(np.abs(wf[r])) if per_row else None
            if per_row:
                assert q[r, k] & 0x7F == 0x7E
        if not per_row:
            assert (q & 0x7F == 0x7E).sum() >= 1
    # an all-zero tensor: finite scale (absmax clamped at 1e-8), all codes zero
    q0, s0 = oracle.quantize_fp8_e4m3(np.zeros((2, 32), np.float16))
    assert np.all(s0 == np.float32(1e-8) / np.float32(448.0)) and not q0.any()


def test_fp8_per_tensor_beats_int8_per_tensor():
    # "FP8, even per tensor, has less error than INT8 per tensor" on weights with outliers
    g = np.random.default_rng(23)
    w = (g.standard_normal((128, 1024)) * 0.02).astype(np.float32)
    w.reshape(-1)[96::97] *= 20
    w = w.astype(np.float16)
    wf = w.astype(np.float64)
    q8, s8 = oracle.quantize_fp8_e4m3(w, per_row=False)
    fp8 = _torch_e4m3_decode(q8).astype(np.float64) * float(s8[0])
    qi, si = oracle.quantize_sym_rows(w.reshape(1, -1), None, 0, 8)
    int8 = (qi.astype(np.float64) * float(si[0])).reshape(w.shape)
    assert _rel(fp8, wf) < _rel(int8, wf)


def test_fp8_gemm_ref_reduces_to_numpy():
    g = np.random.default_rng(24)
    xq = g.integers(0, 256, (5, 64), dtype=np.uint8)
    wq = g.integers(0, 256, (7, 64), dtype=np.uint8)
    xq[(xq & 0x7F) == 0x7F] = 0x10      # no NaN codes
    wq[(wq & 0x7F) == 0x7F] = 0x22
    sx = g.random(5, dtype=np.float32) + 0.5
    sw = g.random(7, dtype=np.float32) + 0.5
    y, b = oracle.gemm_fp8_ref(xq, sx, wq, sw)
    dx, dw = _torch_e4m3_decode(xq).astype(np.float64), _torch_e4m3_decode(wq).astype(np.float64)
    ref = (dx @ dw.T) * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
    assert np.allclose(y, ref, rtol=1e-15, atol=0)
    assert np.allclose(b, (np.abs(dx) @ np.abs(dw).T) * sx[:, None] * sw[None, :], rtol=1e-12)
    # a per-tensor scale (one element) applies to every row
    y1, _ = oracle.gemm_fp8_ref(xq, sx[:1], wq, sw[:1])
    assert np.allclose(y1, (dx @ dw.T) * float(sx[0]) * float(sw[0]), rtol=1e-15)
    ys, _ = oracle.gemm_fp8_ref(xq, sx, wq, sw, ms=[4, 1], ns=[6, 0, 3])
    assert np.array_equal(ys, y[np.ix_([4, 1], [6, 0, 3])])


# --------------------------------------------------------------------------
# LLM.int8() decomposition: reduces to the plain W8A8 and W8A16 references at
# its two extremes, finds planted outlier columns, and beats plain W8A8 on
# activations with outlier features
# --------------------------------------------------------------------------
def _llm_case(seed=31, M=24, N=20, K=256, planted=(3, 70, 71, 200)):
    g = np.random.default_rng(seed)
    x = g.standard_normal((M, K)).astype(np.float32)
    x[:, list(planted)] *= 40.0
    x = x.astype(np.float16)
    w = (g.standard_normal((N, K)) * 0.02).astype(np.float16)
    wq, sw = oracle.quantize_int8_per_channel(w)
    return x, w, wq, sw


def test_outlier_columns_found_and_capped():
    x, _, _, _ = _llm_case()
    idx, total = oracle.outlier_columns(x, 6.0, 16)
    assert total == 4 and list(idx) == [3, 70, 71, 200]
    idx2, total2 = oracle.outlier_columns(x, 6.0, 2)           # cap keeps the lowest columns
    assert total2 == 4 and list(idx2) == [3, 70]
    # the threshold compares max |x| >= t: a column whose max equals t qualifies
    e = np.zeros((2, 16), np.float16)
    e[1, 5], e[0, 9] = 6.0, -5.996
    assert oracle.outlier_columns(e, 6.0, 4) == (np.array([5], np.int32), 1)


def test_llm_int8_reduces_to_w8a8_without_outliers():
    x, _, wq, sw = _llm_case()
    y, b, xq, sx = oracle.llm_int8_ref(x, wq, sw, np.zeros(0, np.int32))
    rxq, rsx = oracle.quantize_int8_per_token(x)
    assert np.array_equal(xq, rxq) and np.array_equal(sx, rsx)
    _, ry, rb = oracle.gemm_w8a8_ref(rxq, rsx, wq, sw)
    assert np.allclose(y, ry, rtol=1e-14, atol=0) and np.allclose(b, rb, rtol=1e-14)


def test_llm_int8_reduces_to_w8a16_with_every_column_carved():
    x, _, wq, sw = _llm_case()
    y, b, xq, _ = oracle.llm_int8_ref(x, wq, sw, np.arange(x.shape[1], dtype=np.int32))
    assert not xq.any()
    ry, rb = oracle.matmul_w8a16_ref(x, wq, sw)
    assert np.allclose(y, ry.T.T, rtol=1e-13, atol=1e-18) and np.allclose(b, rb, rtol=1e-13)


def test_llm_int8_carves_exactly_the_listed_columns():
    x, _, wq, sw = _llm_case()
    idx = np.array([3, 70, 71, 200], np.int32)
    y, _, xq, sx = oracle.llm_int8_ref(x, wq, sw, idx)
    assert not xq[:, idx].any()
    keep = np.ones(x.shape[1], np.float32)
    keep[idx] = 0
    rxq, rsx = oracle.quantize_sym_rows(x, keep, 1, 8)
    assert np.array_equal(xq, rxq) and np.array_equal(sx, rsx)
    # S_out (.) (X_q W_q) + X_16 W_16 written out with numpy in fp64
    xf = x.astype(np.float64)
    w16 = wq[:, idx].astype(np.float64) * sw[:, None]
    ref = (xq.astype(np.float64) @ wq.astype(np.float64).T) * sx[:, None].astype(np.float64) * sw[None, :] \
        + xf[:, idx] @ w16.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-15)
    ys, _, _, _ = oracle.llm_int8_ref(x, wq, sw, idx, ms=[5, 0], ns=[19, 2, 7])
    assert np.array_equal(ys, y[np.ix_([5, 0], [19, 2, 7])])


def test_llm_int8_beats_plain_w8a8_on_outlier_features():
    # carving the outlier dimensions out keeps the other values' precision
    x, w, wq, sw = _llm_case(seed=32, M=64, N=48, K=512, planted=(11, 40, 300))
    exact = x.astype(np.float64) @ (wq.astype(np.float64) * sw[:, None]).T
    idx, _ = oracle.outlier_columns(x, 6.0, 64)
    y_llm, _, _, _ = oracle.llm_int8_ref(x, wq, sw, idx)
    y_w8a8, _, _, _ = oracle.llm_int8_ref(x, wq, sw, np.zeros(0, np.int32))
    assert _rel(y_llm, exact) < 0.5 * _rel(y_w8a8, exact)


# --------------------------------------------------------------------------
# Block-scaled FP4 (MXFP4, NVFP4): E2M1 by brute force over its 16 codes,
# the pages' storage figures, block-scale properties, the GEMM reference
# against numpy on dequantized values
# --------------------------------------------------------------------------
def _e2m1_table():
    return np.array([oracle.e2m1_to_float(c) for c in range(16)], np.float64)


def test_e2m1_codes_and_brute_force_rounding():
    tab = _e2m1_table()
    # "four-bit floats (E2M1)": 8 magnitudes, the largest 6, a sign bit
    assert sorted(set(np.abs(tab))) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert np.array_equal(tab[8:], -tab[:8])
    g = np.random.default_rng(41)
    vals = np.concatenate([g.uniform(-7, 7, 4000), (np.arange(-28, 29) / 4.0)]).astype(np.float32)
    for v in vals:
        code = oracle.float_to_e2m1(v)
        # brute force: the nearest code (within the sign of v); a tie goes to the even mantissa
        cands = range(8, 16) if np.signbit(v) else range(0, 8)
        dist = {c: abs(tab[c] - min(max(v, -6.0), 6.0)) for c in cands}
        best = min(dist.values())
        near = [c for c in cands if dist[c] == best]
        want = near[0] if len(near) == 1 else [c for c in near if c % 2 == 0][0]
        assert code == want, (v, code, want)


def test_fp4_storage_figures_from_the_pages():
    # MXFP4: 32 four-bit values + one 8-bit scale = "about 4.25 bits per weight"
    assert (32 * 4 + 8) / 32 == 4.25
    # NVFP4: 16 values + an FP8 scale: 4.5 bits, "about 3.5 times" smaller than FP16
    assert abs(16 / ((16 * 4 + 8) / 16) - 3.5) < 0.1
    q, s = oracle.quantize_mxfp4(np.zeros((3, 64), np.float16))
    assert q.shape == (3, 32) and s.shape == (3, 2)
    q2, s2, t2 = oracle.quantize_nvfp4(np.zeros((3, 64), np.float16))
    assert q2.shape == (3, 32) and s2.shape == (3, 4) and t2.shape == (1,)


def test_mxfp4_block_scale_rule():
    g = np.random.default_rng(42)
    x = (g.standard_normal((8, 256)) * np.exp(g.uniform(-6, 6, (8, 1)))).astype(np.float16)
    x[0, :32] = 0.0                                                # an all-zero block
    q, s = oracle.quantize_mxfp4(x)
    codes = oracle.unpack_fp4(q, 256)
    tab = _e2m1_table()
    xf = x.astype(np.float64).reshape(8, 8, 32)
    deq = tab[codes].reshape(8, 8, 32) * np.ldexp(1.0, s.astype(np.int64) - 127)[:, :, None]
    amax = np.abs(xf).max(axis=2)
    nz = amax > 0
    # the block maximum lands in [4, 8) units of the shared power of two (so it may saturate to 6)
    ratio = amax[nz] / np.ldexp(1.0, s[nz].astype(np.int64) - 127)
    assert np.all((ratio >= 4) & (ratio < 8))
    assert s[0, 0] == 0 and not codes[0, :32].any()
    # every element is the nearest grid value of the scaled block (saturating at 6)
    scale = np.ldexp(1.0, s.astype(np.int64) - 127)[:, :, None]
    err = np.abs(deq - np.clip(xf, -6 * scale, 6 * scale))
    assert np.all(err <= 1.0 * scale + 1e-300)        # half of the widest step (2 between 4 and 6)


def test_nvfp4_scale_rule_and_error():
    g = np.random.default_rng(43)
    x = (g.standard_normal((6, 128)) * 0.05).astype(np.float32)
    x[:, 5] *= 30
    x = x.astype(np.float16)
    q, s, t = oracle.quantize_nvfp4(x)
    xf = x.astype(np.float64)
    assert t[0] == np.float32(np.float32(np.abs(xf).max()) / np.float32(2688.0))
    sb = np.array([oracle.e4m3_to_float(c) for c in s.reshape(-1)]).reshape(s.shape)
    # the block maximum divided by its decoded scale x tensor scale stays near 6 (E4M3 rounding of the
    # block scale is within 2^-4 relative)
    amax = np.abs(xf).reshape(6, 8, 16).max(axis=2)
    r = amax / (sb * float(t[0]))
    assert np.all((r > 6 / (1 + 2 ** -4) - 1e-9) & (r < 6 / (1 - 2 ** -4) + 1e-9))
    deq = _e2m1_table()[oracle.unpack_fp4(q, 128)].reshape(6, 8, 16) * (sb * float(t[0]))[:, :, None]
    # relative error of the block maximum's quantization: a step of E2M1 near 6 is 2 (1/3 of 6)
    assert np.all(np.abs(deq - xf.reshape(6, 8, 16)) <= (sb * float(t[0]))[:, :, None] * 1.0 + 1e-12)


def test_fp4_gemm_ref_reduces_to_numpy():
    g = np.random.default_rng(44)
    a = (g.standard_normal((5, 128))).astype(np.float16)
    b = (g.standard_normal((7, 128)) * 0.1).astype(np.float16)
    tab = _e2m1_table()
    for nv in (False, True):
        if nv:
            qa, sa, ta = oracle.quantize_nvfp4(a)
            qb, sb, tb = oracle.quantize_nvfp4(b)
            da = np.array([oracle.e4m3_to_float(c) for c in sa.reshape(-1)]).reshape(sa.shape) * float(ta[0])
            db = np.array([oracle.e4m3_to_float(c) for c in sb.reshape(-1)]).reshape(sb.shape) * float(tb[0])
            bs, tav, tbv = 16, float(ta[0]), float(tb[0])
        else:
            qa, sa = oracle.quantize_mxfp4(a)
            qb, sb = oracle.quantize_mxfp4(b)
            da, db = np.ldexp(1.0, sa.astype(np.int64) - 127), np.ldexp(1.0, sb.astype(np.int64) - 127)
            bs, tav, tbv = 32, 1.0, 1.0
        wa = tab[oracle.unpack_fp4(qa, 128)] * np.repeat(da, bs, axis=1)
        wb = tab[oracle.unpack_fp4(qb, 128)] * np.repeat(db, bs, axis=1)
        y, bd = oracle.gemm_fp4_ref(nv, qa, sa, tav, qb, sb, tbv, 128)
        assert np.allclose(y, wa @ wb.T, rtol=1e-12, atol=1e-300)
        assert np.allclose(bd, np.abs(wa) @ np.abs(wb).T, rtol=1e-12)
        # dequantized values approximate the inputs (the format works): relative Frobenius error < 20%
        assert _rel(wa, a.astype(np.float64)) < 0.2
        ys, _ = oracle.gemm_fp4_ref(nv, qa, sa, tav, qb, sb, tbv, 128, ms=[4, 0], ns=[6, 1])
        assert np.array_equal(ys, y[np.ix_([4, 0], [6, 1])])


# --------------------------------------------------------------------------
# GPTQ and AWQ: the Hessian and its factor against numpy, the degenerate cases
# that reduce to round-to-nearest, the objective each method lowers, and the
# pages' direction (GPTQ beats RTN on its calibration data; AWQ's scaling
# helps where input channels carry outliers)
# --------------------------------------------------------------------------
def _calib_case(seed, N=48, K=256, T=384, outlier_channels=(), scale=30.0):
    g = np.random.default_rng(seed)
    x = g.standard_normal((T, K)).astype(np.float32)
    # correlated inputs (a few shared directions) so that compensation has something to use
    x += 0.8 * (g.standard_normal((T, 4)) @ g.standard_normal((4, K))).astype(np.float32)
    for c in outlier_channels:
        x[:, c] *= scale
    w = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    return x.astype(np.float16), w.astype(np.float16)


def _objective(x, w, qw, sc, qz, K, g, s=None):
    what = oracle.dequant_int4(qw, sc, qz, K, g)
    if s is not None:
        what = what / s.astype(np.float64)[None, :]
    d = w.astype(np.float64) - what
    return float(np.sum((x.astype(np.float64) @ d.T) ** 2))


def test_hessian_and_factor_against_numpy():
    x, _ = _calib_case(51, K=64, T=80)
    H = oracle.hessian(x)
    xf = x.astype(np.float64)
    assert np.allclose(H, 2 * xf.T @ xf, rtol=1e-13, atol=1e-10)
    U = oracle.gptq_hinv_chol(H, 0.01)
    Hd = H + 0.01 * np.mean(np.diag(H)) * np.eye(64)
    assert np.allclose(np.triu(U), U)
    assert np.allclose(U.T @ U, np.linalg.inv(Hd), rtol=1e-9, atol=1e-12)
    assert np.allclose(U, np.linalg.cholesky(np.linalg.inv(Hd)).T, rtol=1e-8, atol=1e-12)


def test_gptq_with_identity_hessian_is_round_to_nearest():
    # U = I: no compensation, every block's grid and codes are plain RTN of the weights
    _, w = _calib_case(52)
    K = w.shape[1]
    for g in (64, 128):
        qw, sc, qz = oracle.gptq(w, np.eye(K), g)
        rqw, rsc, rqz = oracle.quantize_group_int4(w, g)
        assert np.array_equal(qw, rqw) and np.array_equal(sc.view(np.uint16), rsc.view(np.uint16))
        assert np.array_equal(qz, rqz)


def test_gptq_lowers_the_calibration_objective():
    x, w = _calib_case(53)
    K = w.shape[1]
    H = oracle.hessian(x)
    U = oracle.gptq_hinv_chol(H, 0.01)
    qw, sc, qz = oracle.gptq(w, U, 128)
    rqw, rsc, rqz = oracle.quantize_group_int4(w, 128)
    e_gptq = _objective(x, w, qw, sc, qz, K, 128)
    e_rtn = _objective(x, w, rqw, rsc, rqz, K, 128)
    # "on its own calibration tokens" GPTQ is well below round-to-nearest
    assert e_gptq < 0.8 * e_rtn


def test_awq_grid_zero_is_round_to_nearest_and_search_picks_the_minimum():
    x, w = _calib_case(54, outlier_channels=(3, 70, 200))
    K = w.shape[1]
    H = oracle.hessian(x)
    qw, sc, qz, s, best, err = oracle.awq(w, x, H, 128, grid=np.array([0.0]))
    rqw, rsc, rqz = oracle.quantize_group_int4(w, 128)
    assert np.all(s == 1.0) and np.array_equal(qw, rqw) and np.array_equal(qz, rqz)
    # the error the search computes is the calibration objective sum_n D H D^T (H = 2 X^T X)
    assert abs(err[0] - 2 * _objective(x, w, rqw, rsc, rqz, K, 128)) <= 1e-9 * err[0]
    qw, sc, qz, s, best, err = oracle.awq(w, x, H, 128)
    assert best == int(np.argmin(err)) and err[best] <= err[0]
    assert abs(2 * _objective(x, w, qw, sc, qz, K, 128, s) - err[best]) <= 1e-9 * err[best]


def test_awq_helps_with_outlier_channels():
    # "AWQ's scaling helps where there are outliers": planted channels 30x the others
    x, w = _calib_case(55, outlier_channels=(3, 70, 200), scale=30.0)
    H = oracle.hessian(x)
    _, _, _, _, best, err = oracle.awq(w, x, H, 128)
    assert best > 0 and err[best] < 0.9 * err[0]


def test_bf16_decode_and_reference_against_torch():
    import torch
    bits = np.arange(65536, dtype=np.uint32)
    ours = np.array([oracle.bf16_to_float(int(b)) for b in bits[::7]], np.float32)
    ref = torch.from_numpy(bits[::7].astype(np.int32).astype(np.int16)).view(torch.bfloat16).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    # the bf16 reference equals the fp16 one on activations exact in both formats
    g = np.random.default_rng(71)
    w = (g.standard_normal((20, 256)) * 0.02).astype(np.float16)
    qw, sc, qz = oracle.quantize_group_int4(w, 128)
    x = (g.integers(-64, 64, (2, 256)) / 8.0).astype(np.float32)         # exact in fp16 and bf16
    xb = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    y16, b16 = oracle.matmul_w4a16_ref(x.astype(np.float16), qw, sc, qz, 256)
    ybf, bbf = oracle.matmul_w4a16_ref_bf16(xb, qw, sc, qz, 256)
    assert np.array_equal(y16, ybf) and np.array_equal(b16, bbf)
