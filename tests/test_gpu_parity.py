"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on seeded inputs.

Codes, scales, zero points, INT8 codes/scales and smoothing factors must be
bit-exact; matmul outputs must satisfy |y - y_ref| <= 2e-3 * sum_k |w^ x| + 1e-5
per element (y_ref and the bound in fp64 from the oracle).  Small cases span
several tiles and ragged tails; the full-size workloads are checked on sampled
rows the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

RTOL_BOUND, ATOL = 2e-3, 1e-5


@pytest.fixture(scope="module")
def wq():
    import bit_gemv_gemm_group_b200 as m
    return m


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t, dtype=None):
    a = t.cpu().numpy()
    return a.view(dtype) if dtype is not None else a


def assert_within_bound(y, y_ref, bound, what=""):
    y = np.asarray(y, np.float64)
    err = np.abs(y - y_ref)
    lim = RTOL_BOUND * bound + ATOL
    bad = err > lim
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst excess "
                           f"{(err - lim).max():.3e} at {np.unravel_index(np.argmax(err - lim), err.shape)}")


def sample_rows(N, k=256, seed=0):
    if N <= k:
        return np.arange(N)
    r = np.random.default_rng(seed).choice(N, size=k - 2, replace=False)
    return np.unique(np.concatenate([r, [0, N - 1]])).astype(np.int32)


# --------------------------------------------------------------------------
# INT4 group quantizer
# --------------------------------------------------------------------------
def _special_weights(N, K, seed, dtype=np.float16):
    g = np.random.default_rng(seed)
    w = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    w.reshape(-1)[96::97] *= 20
    if N > 8 and K >= 512:
        w[1, :128] = 0.0
        w[2, 128:256] = 0.25
        w[3, 256:384] = np.abs(w[3, 256:384]) + 0.01
        w[4, 384:512] = -np.abs(w[4, 384:512]) - 0.01
        w[5, ::7] = 0.0
    if N > 8 and K >= 640:
        # s = 1/16 exactly and every other weight at (k + 1/2) / 16: w / s lands on ties
        tie = (np.arange(128) % 14 + 0.5) / 16.0
        tie[0], tie[1] = 0.0, 15.0 / 16.0
        w[6, 512:640] = tie
    return w.astype(dtype)


SMALL_INT4 = [  # (N, K, g, dtype)
    (1, 128, 128, np.float16), (17, 384, 128, np.float16), (33, 1024, 128, np.float16),
    (64, 1536, 128, np.float16), (9, 96, 32, np.float16), (40, 640, 64, np.float16),
    (13, 2048, 256, np.float16), (24, 512, 128, np.float32), (300, 4096, 128, np.float16),
    (11, 768, 256, np.float16), (13, 4096, 64, np.float16), (9, 8320, 128, np.float16),
    (10, 1280, 128, np.float16),
]


@pytest.mark.parametrize("N,K,g,dtype", SMALL_INT4)
def test_int4_quantizer_bit_exact_small(wq, N, K, g, dtype):
    w = _special_weights(N, K, seed=N * 7 + K, dtype=dtype)
    qw, sc, qz = wq.quantize_group_int4(dev(w), g)
    torch.cuda.synchronize()
    rqw, rsc, rqz = oracle.quantize_group_int4(w, g)
    assert np.array_equal(host(qw, np.uint32), rqw)
    assert np.array_equal(host(sc).view(np.uint16), rsc.view(np.uint16))
    assert np.array_equal(host(qz, np.uint32), rqz)


@pytest.mark.parametrize("cfg,shape_index", [("tiny_w4a16", 0), ("decode_4096", 0), ("mlp_8b", 0), ("mlp_8b", 1),
                                               ("llama70b_class", 0), ("llama70b_class", 1)])
def test_int4_quantizer_bit_exact_configs(wq, cfg, shape_index):
    # The benchmarked 70B-class shapes are quantized in the launch configuration the bench times.
    w = workloads.config_weight(cfg, shape_index)
    qw, sc, qz = wq.quantize_group_int4(dev(w), 128)
    torch.cuda.synchronize()
    rows = sample_rows(w.shape[0], 512, seed=workloads.CONFIGS[cfg].seed)
    rqw, rsc, rqz = oracle.quantize_group_int4(w[rows], 128)
    assert np.array_equal(host(qw, np.uint32)[rows], rqw)
    assert np.array_equal(host(sc).view(np.uint16)[rows], rsc.view(np.uint16))
    assert np.array_equal(host(qz, np.uint32)[rows], rqz)


def test_int4_quantizer_repeatable(wq):
    # The bulk-copy ring reuses shared-memory slots; repeated runs must give the same bits, and
    # the rows of every CTA's first stages (whose slots are refilled) must match the oracle.
    g = np.random.default_rng(7)
    w = (g.standard_normal((4096, 4096)) * 0.02).astype(np.float16)
    wd = dev(w)
    runs = []
    for _ in range(5):
        qw, sc, qz = wq.quantize_group_int4(wd, 128)
        torch.cuda.synchronize()
        runs.append((host(qw, np.uint32), host(sc).view(np.uint16), host(qz, np.uint32)))
    for r in runs[1:]:
        assert all(np.array_equal(a, b) for a, b in zip(runs[0], r))
    rqw, rsc, rqz = oracle.quantize_group_int4(w[:1024], 128)
    assert np.array_equal(runs[0][0][:1024], rqw)
    assert np.array_equal(runs[0][1][:1024], rsc.view(np.uint16))
    assert np.array_equal(runs[0][2][:1024], rqz)


# --------------------------------------------------------------------------
# W4A16 GEMV
# --------------------------------------------------------------------------
GEMV_SMALL = [  # (N, K, g, B)
    (1, 128, 128, 1), (17, 384, 128, 1), (33, 1024, 128, 3), (64, 1536, 128, 8),
    (9, 96, 32, 2), (40, 640, 64, 4), (13, 2048, 256, 5), (300, 4096, 128, 1),
    (3000, 2048, 128, 1), (3000, 2048, 128, 8), (2500, 512, 128, 6), (129, 7168, 128, 7),
    (77, 256, 128, 4), (520, 1280, 128, 2), (4100, 768, 128, 8), (1000, 3328, 128, 3),
]


@pytest.mark.parametrize("N,K,g,B", GEMV_SMALL)
def test_gemv_w4a16_small(wq, N, K, g, B):
    w = _special_weights(N, K, seed=N + 3 * K)
    rqw, rsc, rqz = oracle.quantize_group_int4(w, g)
    x = workloads.activations(B, K, 0.01, 50.0, seed=N, tensor_id=K)
    x[0, :3] = 0.0
    y = wq.gemv_w4a16(dev(x), dev(rqw.view(np.int32)), dev(rsc), dev(rqz.view(np.int32)), g)
    torch.cuda.synchronize()
    y_ref, bound = oracle.matmul_w4a16_ref(x, rqw, rsc, rqz, K, g)
    assert_within_bound(host(y).astype(np.float64), y_ref, bound, f"gemv N={N} K={K} B={B}")


@pytest.mark.parametrize("N,K,B", [(520, 2048, 1), (520, 2048, 8), (3000, 2048, 4)])
def test_gemv_w4a16_small_activations(wq, N, K, B):
    # Activations of magnitude 1e-4: half of the streaming kernel's products take x * 2^-4
    # rounded in fp16 (inexact below 2^-10); the roundings cancel and stay inside the tolerance.
    w = workloads.weight_normal(N, K, 0.02, seed=11, tensor_id=N)
    rqw, rsc, rqz = oracle.quantize_group_int4(w, 128)
    x = workloads.activations(B, K, 0.0, 1.0, seed=K, tensor_id=B).astype(np.float32) * np.float32(1e-4)
    x = x.astype(np.float16)
    y = wq.gemv_w4a16(dev(x), dev(rqw.view(np.int32)), dev(rsc), dev(rqz.view(np.int32)), 128)
    torch.cuda.synchronize()
    y_ref, bound = oracle.matmul_w4a16_ref(x, rqw, rsc, rqz, K, 128)
    assert_within_bound(host(y).astype(np.float64), y_ref, bound, f"gemv small x N={N} K={K} B={B}")


# Rows of one tiny value accumulate every rounding the same way, so they expose any inexact
# step on the activations; 56 * 2^-24 and 2^-22 are fp16 subnormals.  The four paths are the
# batch-1 and batch-8 GEMV (streaming kernel, one n-tile) and the 16- and 32-row GEMM (two
# n-tiles, one and two passes).
TINY_VALUES = [56 * 2.0 ** -24, 1e-6, 2.0 ** -22, 1e-4]
TINY_PATHS = [("gemv", 1), ("gemv", 8), ("gemm", 16), ("gemm", 32)]


def _run_w4(wq, kind, x, rqw, rsc, rqz, g=128):
    f = wq.gemv_w4a16 if kind == "gemv" else wq.gemm_w4a16
    y = f(dev(x), dev(rqw.view(np.int32)), dev(rsc), dev(rqz.view(np.int32)), g)
    torch.cuda.synchronize()
    return host(y).astype(np.float64)


@pytest.mark.parametrize("value", TINY_VALUES)
@pytest.mark.parametrize("kind,B", TINY_PATHS)
def test_w4a16_constant_tiny_activations(wq, value, kind, B):
    N, K = 256, 2048
    w = workloads.weight_normal(N, K, 0.02, seed=12, tensor_id=N)
    rqw, rsc, rqz = oracle.quantize_group_int4(w, 128)
    x = np.full((B, K), value, np.float16)
    x[B - 1] = -x[B - 1]
    y = _run_w4(wq, kind, x, rqw, rsc, rqz)
    y_ref, bound = oracle.matmul_w4a16_ref(x, rqw, rsc, rqz, K, 128)
    assert_within_bound(y, y_ref, bound, f"{kind} B={B} constant x={value:g}")


@pytest.mark.parametrize("kind,B", TINY_PATHS)
def test_w4a16_mixed_magnitude_activations(wq, kind, B):
    # Per row: groups of ordinary values, groups of random subnormals, groups mixing the two, a
    # group with values up to 4000 beside tiny ones (the fragments carry 16 x there), and one
    # with 30000 beside tiny ones (16 x would overflow; the small values keep x * 2^-4).
    N, K = 300, 2048
    w = workloads.weight_normal(N, K, 0.02, seed=13, tensor_id=N)
    rqw, rsc, rqz = oracle.quantize_group_int4(w, 128)
    g = np.random.default_rng(B)
    x = g.standard_normal((B, K)).astype(np.float32)
    sub = (g.integers(1, 1024, (B, K)) * 2.0 ** -24 * np.where(g.random((B, K)) < 0.5, -1, 1)).astype(np.float32)
    x[:, 128:384] = sub[:, 128:384]
    x[:, 384:512:3] = sub[:, 384:512:3]
    x[:, 512:640] = sub[:, 512:640]
    x[:, 512:640:17] = 4000.0
    x[:, 640:768] = sub[:, 640:768]
    x[:, 640] = 30000.0
    x = x.astype(np.float16)
    y = _run_w4(wq, kind, x, rqw, rsc, rqz)
    y_ref, bound = oracle.matmul_w4a16_ref(x, rqw, rsc, rqz, K, 128)
    assert_within_bound(y, y_ref, bound, f"{kind} B={B} mixed magnitudes")


@pytest.mark.parametrize("cfg", ["tiny_w4a16", "decode_4096", "mlp_8b", "llama70b_class"])
def test_gemv_w4a16_configs(wq, cfg):
    c = workloads.CONFIGS[cfg]
    for si, (N, K) in enumerate(c.shapes):
        w = workloads.config_weight(cfg, si)
        qw, sc, qz = wq.quantize_group_int4(dev(w), 128)
        rows = sample_rows(N, 384, seed=si)
        hqw, hsc, hqz = host(qw, np.uint32), host(sc), host(qz, np.uint32)
        for B in [b for b in c.batches if b <= 8]:
            x = workloads.config_activations(cfg, B, K)
            y = wq.gemv_w4a16(dev(x), qw, sc, qz, 128)
            torch.cuda.synchronize()
            y_ref, bound = oracle.matmul_w4a16_ref(x, hqw, hsc, hqz, K, 128, rows=rows)
            assert_within_bound(host(y).astype(np.float64)[:, rows], y_ref, bound, f"{cfg} {N}x{K} B={B}")


@pytest.mark.parametrize("N,K,B", [(40000, 2048, 1), (30000, 4096, 8), (9000, 14336, 3)])
def test_gemv_w4a16_large_shapes_tile_boundaries(wq, N, K, B):
    # Larger streaming-GEMV shapes (several tiles, K splits over clusters of 1, 2 and 7 CTAs);
    # sampled rows include the rows next to the boundaries of 224- and 128-row tiles and of
    # near-equal row blocks.
    g = np.random.default_rng(N + K)
    w = (g.standard_normal((N, K)) * 0.02).astype(np.float16)
    qw, sc, qz = wq.quantize_group_int4(dev(w), 128)
    bounds = {int(p * N // P) + d for s in range(1, 9) for P in [296 // s] for p in range(1, P)
              for d in (-1, 0)}
    bounds |= {t * r + d for r in (224, 128) for t in range(1, N // r + 1) for d in (-1, 0)}
    rows = np.unique(np.concatenate([sample_rows(N, 256, seed=N), np.array(sorted(bounds), np.int32)]))
    rows = rows[(rows >= 0) & (rows < N)].astype(np.int32)
    x = workloads.activations(B, K, 0.01, 50.0, seed=B, tensor_id=N)
    y = wq.gemv_w4a16(dev(x), qw, sc, qz, 128)
    torch.cuda.synchronize()
    y_ref, bound = oracle.matmul_w4a16_ref(x, host(qw, np.uint32), host(sc), host(qz, np.uint32), K, 128, rows=rows)
    assert_within_bound(host(y).astype(np.float64)[:, rows], y_ref, bound, f"{N}x{K} B={B}")


# --------------------------------------------------------------------------
# INT8 quantizers and smoothing
# --------------------------------------------------------------------------
INT8_SMALL = [(1, 16), (7, 48), (33, 2048), (5, 2064), (64, 4096), (3, 4112), (6, 6000), (9, 8192), (3, 16384),
              (2, 16400), (4, 40960), (5, 28672), (3, 32768), (2, 24592)]


@pytest.mark.parametrize("R,K", INT8_SMALL)
@pytest.mark.parametrize("smoothing", [False, True])
def test_int8_quantizers_bit_exact_small(wq, R, K, smoothing):
    g = np.random.default_rng(R * K)
    a = (g.standard_normal((R, K)) * 2).astype(np.float32)
    a[:, g.choice(K, size=max(1, K // 100), replace=False)] *= 40
    if R > 2:
        a[1] = 0.0
    a = a.astype(np.float16)
    s = (np.exp(g.normal(0, 1, K)) + 0.05).astype(np.float32) if smoothing else None
    sd = dev(s) if smoothing else None
    qc, sc = wq.quantize_int8_per_channel(dev(a), sd)
    qt, st = wq.quantize_int8_per_token(dev(a), sd)
    torch.cuda.synchronize()
    rqc, rsc = oracle.quantize_int8_per_channel(a, s)
    rqt, rst = oracle.quantize_int8_per_token(a, s)
    assert np.array_equal(host(qc), rqc) and np.array_equal(host(sc).view(np.uint32), rsc.view(np.uint32))
    assert np.array_equal(host(qt), rqt) and np.array_equal(host(st).view(np.uint32), rst.view(np.uint32))


SMOOTH_SMALL = [(1, 1, 8), (3, 5, 24), (37, 300, 520), (256, 257, 256), (600, 90, 1032)]


@pytest.mark.parametrize("M,N,K", SMOOTH_SMALL)
@pytest.mark.parametrize("alpha", [0.5, 0.75, 0.0, 1.0])
def test_smooth_small(wq, M, N, K, alpha):
    g = np.random.default_rng(M + N + K)
    X = g.standard_normal((M, K)).astype(np.float32)
    X[:, g.choice(K, size=max(1, K // 50), replace=False)] *= 60
    X[:, 0] = 0.0                                   # an all-zero column hits the 1e-5 clamp
    X = X.astype(np.float16)
    W = (g.standard_normal((N, K)) * 0.02).astype(np.float16)
    s = host(wq.smooth(dev(X), dev(W), alpha))
    ref = oracle.smooth_factors(X, W, alpha)
    if alpha in (0.5, 1.0, 0.0):
        # 0.5: correctly rounded square roots; 1.0 / 0.0: pow(x, 1) and pow(x, 0) are exact
        assert np.array_equal(s.view(np.uint32), ref.view(np.uint32))
    else:
        # fp64 pow rounded to fp32 on both sides: at most 1 ulp apart
        ulps = np.abs(s.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
        assert ulps.max() <= 1


def test_smooth_reuses_dirty_workspace(wq):
    g = np.random.default_rng(5)
    X = g.standard_normal((64, 512)).astype(np.float16)
    W = (g.standard_normal((96, 512)) * 0.02).astype(np.float16)
    ws = torch.full((wq.smooth_workspace_bytes(512),), 0x7f, dtype=torch.uint8, device="cuda")
    s1 = host(wq.smooth(dev(X), dev(W), 0.5, workspace=ws))
    s2 = host(wq.smooth(dev(X), dev(W), 0.5, workspace=ws))
    ref = oracle.smooth_factors(X, W, 0.5)
    assert np.array_equal(s1, ref) and np.array_equal(s2, ref)


# --------------------------------------------------------------------------
# W8A16 GEMV
# --------------------------------------------------------------------------
@pytest.mark.parametrize("N,K,B", [(1, 16, 1), (17, 48, 2), (300, 4096, 1), (3000, 2048, 8), (129, 7168, 5)])
def test_gemv_w8a16_small(wq, N, K, B):
    g = np.random.default_rng(N + K + B)
    w = (g.standard_normal((N, K)) * 0.02).astype(np.float16)
    q, s = oracle.quantize_int8_per_channel(w)
    x = workloads.activations(B, K, 0.01, 50.0, seed=N, tensor_id=B)
    y = host(wq.gemv_w8a16(dev(x), dev(q), dev(s)))
    y_ref, bound = oracle.matmul_w8a16_ref(x, q, s)
    assert_within_bound(y.astype(np.float64), y_ref, bound, f"w8a16 N={N} K={K} B={B}")


def test_w8a16_mlp_8b(wq):
    c = workloads.CONFIGS["mlp_8b"]
    for si, (N, K) in enumerate(c.shapes):
        w = workloads.config_weight("mlp_8b", si)
        q, s = wq.quantize_int8_per_channel(dev(w))
        rows = sample_rows(N, 256, seed=si)
        rq, rs = oracle.quantize_int8_per_channel(w[rows])
        hq, hs = host(q), host(s)
        assert np.array_equal(hq[rows], rq) and np.array_equal(hs[rows].view(np.uint32), rs.view(np.uint32))
        for B in (1, 8):
            x = workloads.config_activations("mlp_8b", B, K)
            y = host(wq.gemv_w8a16(dev(x), q, s))
            y_ref, bound = oracle.matmul_w8a16_ref(x, hq, hs, rows=rows)
            assert_within_bound(y.astype(np.float64)[:, rows], y_ref, bound, f"w8a16 mlp_8b {N}x{K} B={B}")


# --------------------------------------------------------------------------
# W8A8 INT8 tensor-core GEMM
# --------------------------------------------------------------------------
def _gemm_check(wq, xq, sx, wq8, sw, ms=None, ns=None):
    y, acc = wq.gemm_w8a8(dev(xq), dev(sx), dev(wq8), dev(sw), return_acc=True)
    torch.cuda.synchronize()
    racc, ry, rb = oracle.gemm_w8a8_ref(xq, sx, wq8, sw, ms, ns)
    hy, hacc = host(y).astype(np.float64), host(acc).astype(np.int64)
    if ms is not None:
        hy, hacc = hy[np.ix_(ms, ns)], hacc[np.ix_(ms, ns)]
    assert np.array_equal(hacc, racc)
    assert_within_bound(hy, ry, rb, "w8a8")


W8A8_SMALL = [(1, 1, 16), (128, 256, 128), (130, 300, 144), (64, 40, 1040), (257, 513, 256), (300, 1000, 2000),
              (512, 1024, 4096)]


@pytest.mark.parametrize("M,N,K", W8A8_SMALL)
def test_gemm_w8a8_small(wq, M, N, K):
    g = np.random.default_rng(M * N + K)
    xq = g.integers(-128, 128, (M, K), dtype=np.int8)
    wq8 = g.integers(-128, 128, (N, K), dtype=np.int8)
    sx = (g.random(M, dtype=np.float32) + 0.01) * 0.05
    sw = (g.random(N, dtype=np.float32) + 0.01) * 0.01
    _gemm_check(wq, xq, sx, wq8, sw)


def test_gemm_w8a8_every_code_pair(wq):
    # acc[m][n] = (m - 128) * (n - 128): all 256 x 256 int8 products through the tensor cores
    codes = np.arange(-128, 128, dtype=np.int8)
    xq = np.zeros((256, 16), np.int8)
    xq[:, 0] = codes
    wq8 = np.zeros((256, 16), np.int8)
    wq8[:, 5] = codes
    wq8[:, 0] = codes
    _gemm_check(wq, xq, np.ones(256, np.float32), wq8, np.ones(256, np.float32) * np.float32(2 ** -16))


def test_gemm_w8a8_extreme_accumulators(wq):
    K = 8192
    xq = np.full((130, K), -128, np.int8)
    xq[1] = 127
    wq8 = np.full((260, K), -128, np.int8)
    wq8[3, ::2] = 127
    _gemm_check(wq, xq, np.full(130, 1e-6, np.float32), wq8, np.full(260, 1e-4, np.float32))


def test_w8a8_smoothquant_pipeline_full_size(wq):
    # The W8A8 SmoothQuant layer: smoothing -> per-channel(W * s) -> per-token(X / s) -> INT8 GEMM, in the
    # launch configuration the benchmark times; sampled rows checked one by one.
    M, N, K = 2048, 8192, 8192
    X = workloads.config_activations("w8a8_smoothquant", M, K)
    W = workloads.config_weight("w8a8_smoothquant")
    Xd, Wd = dev(X), dev(W)
    s = wq.smooth(Xd, Wd, 0.5)
    wq8, sw = wq.quantize_int8_per_channel(Wd, s)
    xq8, sx = wq.quantize_int8_per_token(Xd, s)
    y, acc = wq.gemm_w8a8(xq8, sx, wq8, sw, return_acc=True)
    torch.cuda.synchronize()
    rs = oracle.smooth_factors(X, W, 0.5)
    assert np.array_equal(host(s).view(np.uint32), rs.view(np.uint32))
    ms = sample_rows(M, 96, seed=1)
    ns = sample_rows(N, 160, seed=2)
    rxq, rsx = oracle.quantize_int8_per_token(X[ms], rs)
    rwq, rsw = oracle.quantize_int8_per_channel(W[ns], rs)
    assert np.array_equal(host(xq8)[ms], rxq) and np.array_equal(host(sx)[ms], rsx)
    assert np.array_equal(host(wq8)[ns], rwq) and np.array_equal(host(sw)[ns], rsw)
    racc, ry, rb = oracle.gemm_w8a8_ref(rxq, rsx, rwq, rsw)
    assert np.array_equal(host(acc)[np.ix_(ms, ns)].astype(np.int64), racc)
    assert_within_bound(host(y)[np.ix_(ms, ns)].astype(np.float64), ry, rb, "w8a8_smoothquant")
    assert wq.device_status() == 0


# --------------------------------------------------------------------------
# W4A16 tensor-core GEMM
# --------------------------------------------------------------------------
GEMM_W4_SMALL = [  # (M, N, K): ragged M/N, K on and off the 1024-code fast path, split-K clusters
    (16, 128, 128), (16, 300, 1024), (20, 256, 2048), (64, 1000, 4096), (33, 129, 1152),
    (128, 512, 8192), (100, 384, 3072), (16, 4096, 14336), (48, 640, 16384), (17, 130, 640),
    (200, 384, 2048), (300, 260, 1024),  # two and three 128-row activation tiles, ragged
    (12, 300, 1280), (25, 520, 2304),  # 9..15 rows in one streaming pass; 16 + 9 rows
]


@pytest.mark.parametrize("M,N,K", GEMM_W4_SMALL)
def test_gemm_w4a16_small(wq, M, N, K):
    w = _special_weights(N, K, seed=M + N + K)
    rqw, rsc, rqz = oracle.quantize_group_int4(w, 128)
    x = workloads.activations(M, K, 0.01, 50.0, seed=M, tensor_id=N)
    y = wq.gemm_w4a16(dev(x), dev(rqw.view(np.int32)), dev(rsc), dev(rqz.view(np.int32)), 128)
    torch.cuda.synchronize()
    rows = sample_rows(N, 300, seed=K)
    y_ref, bound = oracle.matmul_w4a16_ref(x, rqw, rsc, rqz, K, 128, rows=rows)
    assert_within_bound(host(y).astype(np.float64)[:, rows], y_ref, bound, f"gemm_w4a16 M={M} N={N} K={K}")
    assert wq.device_status() == 0


GEMM_W4_GROUPS = [  # (M, N, K, g): the group sizes the quantizer writes, ragged M/N, split-K, M < 16
    (16, 300, 1024, 32), (64, 1000, 4096, 64), (100, 384, 3072, 256), (130, 260, 2048, 32),
    (48, 640, 16384, 64), (12, 300, 1280, 256), (9, 130, 640, 32), (33, 129, 1152, 64),
]


@pytest.mark.parametrize("M,N,K,g", GEMM_W4_GROUPS)
def test_gemm_w4a16_group_sizes(wq, M, N, K, g):
    # A layout wq_quantize_group_int4 writes is one wq_gemm_w4a16 consumes, for every group size.
    w = _special_weights(N, K, seed=M + N + K + g)
    qw, sc, qz = wq.quantize_group_int4(dev(w), g)
    x = workloads.activations(M, K, 0.01, 50.0, seed=M + g, tensor_id=N)
    y = wq.gemm_w4a16(dev(x), qw, sc, qz, g)
    torch.cuda.synchronize()
    rqw, rsc, rqz = oracle.quantize_group_int4(w, g)
    assert np.array_equal(host(qw, np.uint32), rqw) and np.array_equal(host(qz, np.uint32), rqz)
    rows = sample_rows(N, 300, seed=K)
    y_ref, bound = oracle.matmul_w4a16_ref(x, rqw, rsc, rqz, K, g, rows=rows)
    assert_within_bound(host(y).astype(np.float64)[:, rows], y_ref, bound, f"gemm_w4a16 g={g} M={M} N={N} K={K}")
    assert wq.device_status() == 0


@pytest.mark.parametrize("cfg", ["mlp_8b", "llama70b_class"])
def test_gemm_w4a16_configs(wq, cfg):
    c = workloads.CONFIGS[cfg]
    for si, (N, K) in enumerate(c.shapes):
        w = workloads.config_weight(cfg, si)
        qw, sc, qz = wq.quantize_group_int4(dev(w), 128)
        del w
        rows = sample_rows(N, 128, seed=si + 10)
        hqw, hsc, hqz = host(qw, np.uint32), host(sc), host(qz, np.uint32)
        for B in c.batches:
            x = workloads.config_activations(cfg, B, K)
            y = wq.matmul_w4a16(dev(x), qw, sc, qz, 128)
            torch.cuda.synchronize()
            y_ref, bound = oracle.matmul_w4a16_ref(x, hqw[rows], hsc[rows], hqz[rows], K, 128)
            assert_within_bound(host(y).astype(np.float64)[:, rows], y_ref, bound, f"{cfg} {N}x{K} B={B}")
    assert wq.device_status() == 0


# --------------------------------------------------------------------------
# Determinism at full size: every launch of a kernel on the same inputs gives
# the same bits.  This holds at any size; a race between a ring slot's release
# and its refill would show up as a difference somewhere in the output.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("shape_index", [0, 1])
def test_w4a16_matmuls_repeat_bit_identically(wq, shape_index):
    w = workloads.config_weight("llama70b_class", shape_index)
    N, K = w.shape
    qw, sc, qz = wq.quantize_group_int4(dev(w), 128)
    del w
    for B in (1, 16, 64):
        x = dev(workloads.config_activations("llama70b_class", B, K))
        first = wq.matmul_w4a16(x, qw, sc, qz, 128)
        for _ in range(3):
            again = wq.matmul_w4a16(x, qw, sc, qz, 128)
            torch.cuda.synchronize()
            assert torch.equal(first.view(torch.int16), again.view(torch.int16)), f"{N}x{K} B={B}"
    assert wq.device_status() == 0


# --------------------------------------------------------------------------
# FP8 E4M3 W8A8: quantizer bit-exact, tensor-core GEMM within the tolerance
# --------------------------------------------------------------------------
FP8_Q_SMALL = [(1, 16), (7, 48), (33, 2048), (5, 2064), (64, 4096), (3, 16384), (2, 16400), (4, 40960), (300, 1024)]


@pytest.mark.parametrize("R,K", FP8_Q_SMALL)
@pytest.mark.parametrize("per_row", [True, False])
def test_fp8_quantizer_bit_exact_small(wq, R, K, per_row):
    g = np.random.default_rng(R * K + per_row)
    a = (g.standard_normal((R, K)) * 2).astype(np.float32)
    a[:, g.choice(K, size=max(1, K // 100), replace=False)] *= 40
    if R > 2:
        a[1] = 0.0                                        # an all-zero row: the 1e-8 clamp (per row)
        a[2, : K // 2] *= 1e-6                            # E4M3 subnormals and values that round to 0
    a = a.astype(np.float16)
    q, s = wq.quantize_fp8_e4m3(dev(a), per_row=per_row)
    torch.cuda.synchronize()
    rq, rs = oracle.quantize_fp8_e4m3(a, per_row=per_row)
    assert np.array_equal(host(s).view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(host(q), rq)


def test_fp8_quantizer_every_e4m3_midpoint(wq):
    # x / s placed next to every E4M3 rounding boundary (both sides and on it): the decisions
    # that the fast path hands to the IEEE quotient
    fin = np.array([oracle.e4m3_to_float(c) for c in range(0x7F)], np.float64)
    mids = (fin[:-1] + fin[1:]) / 2
    vals = np.concatenate([mids, mids * (1 + 2 ** -10), mids * (1 - 2 ** -10), fin])
    K = 16 * ((vals.size + 15) // 16)
    row = np.zeros(K, np.float64)
    row[: vals.size] = vals
    a = np.stack([row, -row]).astype(np.float16)          # scale 448 / 448: x / s is x
    a[:, -1] = 448.0
    q, s = wq.quantize_fp8_e4m3(dev(a), per_row=True)
    torch.cuda.synchronize()
    rq, rs = oracle.quantize_fp8_e4m3(a, per_row=True)
    assert np.array_equal(host(s), rs) and np.array_equal(host(q), rq)


def _fp8_gemm_check(wq, xq, sx, wq8, sw, ms=None, ns=None):
    y = wq.gemm_fp8(dev(xq), dev(sx), dev(wq8), dev(sw))
    torch.cuda.synchronize()
    ry, rb = oracle.gemm_fp8_ref(xq, sx, wq8, sw, ms, ns)
    hy = host(y).astype(np.float64)
    if ms is not None:
        hy = hy[np.ix_(ms, ns)]
    assert_within_bound(hy, ry, rb, "fp8 gemm")


def _random_e4m3(g, shape):
    c = g.integers(0, 256, shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x3A                          # no NaN codes
    return c


FP8_GEMM_SMALL = [(1, 1, 16), (128, 256, 128), (130, 300, 144), (64, 40, 1040), (257, 513, 256),
                  (300, 1000, 2000), (512, 1024, 4096)]


@pytest.mark.parametrize("M,N,K", FP8_GEMM_SMALL)
def test_gemm_fp8_small(wq, M, N, K):
    g = np.random.default_rng(M * N + K + 1)
    xq, wq8 = _random_e4m3(g, (M, K)), _random_e4m3(g, (N, K))
    sx = (g.random(M, dtype=np.float32) + 0.01) * 0.05
    sw = (g.random(N, dtype=np.float32) + 0.01) * 0.01
    _fp8_gemm_check(wq, xq, sx, wq8, sw)
    _fp8_gemm_check(wq, xq, sx[:1], wq8, sw[:1])           # per-tensor scales


def test_gemm_fp8_every_code_pair(wq):
    # acc[m][n] = e4m3(m) * e4m3(n): every product of two finite E4M3 codes
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    xq = np.zeros((codes.size, 16), np.uint8)
    xq[:, 0] = codes
    wq8 = np.zeros((codes.size, 16), np.uint8)
    wq8[:, 0] = codes
    y, acc = wq.gemm_fp8(dev(xq), dev(np.ones(1, np.float32)), dev(wq8), dev(np.ones(1, np.float32)),
                         return_acc=True)
    torch.cuda.synchronize()
    dec = np.array([oracle.e4m3_to_float(c) for c in codes], np.float64)
    assert np.array_equal(host(acc).astype(np.float64), np.outer(dec, dec))


def test_fp8_w8a8_pipeline_full_size(wq):
    # The W8A8 layer in FP8: per-token activations, per-channel weights (and the per-tensor
    # variant of the listing), tensor-core GEMM; sampled rows checked one by one.
    M, N, K = 2048, 8192, 8192
    X = workloads.config_activations("w8a8_smoothquant", M, K)
    W = workloads.config_weight("w8a8_smoothquant")
    ms = sample_rows(M, 64, seed=3)
    ns = sample_rows(N, 96, seed=4)
    for per_row in (True, False):
        xq, sx = wq.quantize_fp8_e4m3(dev(X), per_row=per_row)
        w8, sw = wq.quantize_fp8_e4m3(dev(W), per_row=per_row)
        y = wq.gemm_fp8(xq, sx, w8, sw)
        torch.cuda.synchronize()
        hxq, hsx, hw8, hsw = host(xq), host(sx), host(w8), host(sw)
        if per_row:
            rxq, rsx = oracle.quantize_fp8_e4m3(X[ms], per_row=True)
            rwq, rsw = oracle.quantize_fp8_e4m3(W[ns], per_row=True)
            assert np.array_equal(hxq[ms], rxq) and np.array_equal(hsx[ms], rsx)
            assert np.array_equal(hw8[ns], rwq) and np.array_equal(hsw[ns], rsw)
        else:  # one scale over the whole tensor: the oracle quantizes all of it
            rxq, rsx = oracle.quantize_fp8_e4m3(X, per_row=False)
            rwq, rsw = oracle.quantize_fp8_e4m3(W, per_row=False)
            assert np.array_equal(hsx, rsx) and np.array_equal(hsw, rsw)
            assert np.array_equal(hxq, rxq) and np.array_equal(hw8, rwq)
            del rxq, rwq
        ry, rb = oracle.gemm_fp8_ref(hxq, hsx, hw8, hsw, ms, ns)
        assert_within_bound(host(y)[np.ix_(ms, ns)].astype(np.float64), ry, rb, f"fp8 per_row={per_row}")
    assert wq.device_status() == 0


# --------------------------------------------------------------------------
# LLM.int8() decomposition: outlier columns and codes bit-exact, the fused
# GEMM (INT8 tensor cores + 16-bit outlier product in the epilogue) within
# the tolerance
# --------------------------------------------------------------------------
def _llm_inputs(M, N, K, planted, seed, scale=40.0):
    g = np.random.default_rng(seed)
    x = g.standard_normal((M, K)).astype(np.float32)
    x[:, list(planted)] *= scale
    x = x.astype(np.float16)
    w = (g.standard_normal((N, K)) * 0.02).astype(np.float16)
    wq8, sw = oracle.quantize_int8_per_channel(w)
    return x, wq8, sw


LLM_SMALL = [  # (M, N, K, planted columns, cap)
    (1, 1, 16, (3,), 16), (128, 256, 128, (0, 127), 16), (130, 300, 144, (5, 6, 7, 100), 16),
    (64, 40, 1040, tuple(range(0, 1040, 41)), 32), (257, 513, 256, (), 16), (300, 1000, 2000, (7, 1999), 64),
    (200, 260, 512, tuple(range(3, 512, 9)), 48),  # 57 outlier columns, 48 carved: the rest stay INT8
]


@pytest.mark.parametrize("M,N,K,planted,cap", LLM_SMALL)
def test_llm_int8_small(wq, M, N, K, planted, cap):
    x, wq8, sw = _llm_inputs(M, N, K, planted, seed=M + N + K)
    xd, wd, sd = dev(x), dev(wq8), dev(sw)
    idx, count, keep = wq.outlier_columns(xd, 6.0, cap)
    xq, sx = wq.quantize_int8_per_channel(xd, keep)
    x16, w16 = wq.gather_outliers(xd, wd, idx, count, cap)
    y = wq.gemm_w8a8_outliers(xq, sx, wd, sd, x16, w16)
    torch.cuda.synchronize()
    ridx, total = oracle.outlier_columns(x, 6.0, cap)
    assert int(host(count)[0]) == total
    assert np.array_equal(host(idx)[: ridx.size], ridx)
    assert np.all(host(idx)[ridx.size:] == 0)  # the unused entries are written too
    assert np.array_equal(host(keep) == 0, np.isin(np.arange(K), ridx))
    ry, rb, rxq, rsx = oracle.llm_int8_ref(x, wq8, sw, ridx)
    assert np.array_equal(host(xq), rxq) and np.array_equal(host(sx), rsx)
    hx16, hw16 = host(x16), host(w16)
    assert np.array_equal(hx16[:, : ridx.size], x[:, ridx]) and not hx16[:, ridx.size:].any()
    assert np.array_equal(hw16[:, : ridx.size], wq8[:, ridx].astype(np.float16)) and not hw16[:, ridx.size:].any()
    assert_within_bound(host(y).astype(np.float64), ry, rb, f"llm.int8 M={M} N={N} K={K}")
    assert wq.device_status() == 0


def test_llm_int8_split_last_round(wq):
    # 160 tiles of 128 x 256 on 148 SMs: the last 12 are shared by CTA pairs (each half of K, the
    # halves summed through distributed shared memory), and their epilogue adds the outlier product.
    M, N, K = 1280, 4096, 512
    x, wq8, sw = _llm_inputs(M, N, K, tuple(range(5, K, 37)), seed=23)
    xd, wd, sd = dev(x), dev(wq8), dev(sw)
    y, count = wq.llm_int8_matmul(xd, wd, sd, 6.0, 16)
    torch.cuda.synchronize()
    ridx, total = oracle.outlier_columns(x, 6.0, 16)
    assert int(host(count)[0]) == total
    ms = np.arange(M, dtype=np.int32)
    ns = np.arange(14 * 256, 16 * 256, dtype=np.int32)
    ry, rb, _, _ = oracle.llm_int8_ref(x, wq8, sw, ridx, ms, ns)
    assert_within_bound(host(y)[:, ns].astype(np.float64), ry, rb, "llm.int8 split round")
    ms2, ns2 = sample_rows(M, 64, seed=5), sample_rows(N, 64, seed=6)
    ry2, rb2, _, _ = oracle.llm_int8_ref(x, wq8, sw, ridx, ms2, ns2)
    assert_within_bound(host(y)[np.ix_(ms2, ns2)].astype(np.float64), ry2, rb2, "llm.int8 split sample")
    assert wq.device_status() == 0


def test_llm_int8_full_size(wq):
    # The W8A8 layer's activations (64 outlier channels x60) through the whole sequence at
    # threshold 6: the 64 planted columns are carved out; sampled rows checked one by one.
    M, N, K = 2048, 8192, 8192
    X = workloads.config_activations("w8a8_smoothquant", M, K)
    W = workloads.config_weight("w8a8_smoothquant")
    wq8, sw = wq.quantize_int8_per_channel(dev(W))
    y, count = wq.llm_int8_matmul(dev(X), wq8, sw, 6.0, 64)
    torch.cuda.synchronize()
    ridx, total = oracle.outlier_columns(X, 6.0, 64)
    assert int(host(count)[0]) == total == 64
    ms = sample_rows(M, 64, seed=5)
    ns = sample_rows(N, 96, seed=6)
    ry, rb, _, _ = oracle.llm_int8_ref(X, host(wq8), host(sw), ridx, ms=ms, ns=ns)
    assert_within_bound(host(y)[np.ix_(ms, ns)].astype(np.float64), ry, rb, "llm.int8 full size")
    assert wq.device_status() == 0


# --------------------------------------------------------------------------
# Block-scaled FP4 (MXFP4, NVFP4): quantizers bit-exact, tcgen05 block-scaled
# GEMM within the tolerance
# --------------------------------------------------------------------------
FP4_Q_SMALL = [(1, 32), (7, 64), (33, 2048), (5, 2080), (64, 4096), (3, 16384), (300, 1024)]


def _sf_offsets(R, F):
    # byte offset of factor f of row r in the tensor-core atom layout (see wq.h)
    r = np.arange(R)[:, None]
    f = np.arange(F)[None, :]
    fg = -(-F // 4)
    return ((r >> 7) * fg + (f >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (f & 3)


def sf_to_atoms(sf):
    """Row-major scale factors [R][F] -> the atom-layout buffer the GPU kernels use."""
    R, F = sf.shape
    out = np.zeros(-(-R // 128) * -(-F // 4) * 512, np.uint8)
    out[_sf_offsets(R, F)] = sf
    return out


def sf_from_atoms(buf, R, F):
    """The atom-layout buffer -> row-major scale factors [R][F]."""
    return np.asarray(buf)[_sf_offsets(R, F)]


def test_sf_atom_layout_helpers_round_trip():
    g = np.random.default_rng(3)
    sf = g.integers(0, 256, (300, 37), dtype=np.uint8)
    buf = sf_to_atoms(sf)
    assert buf.size == 3 * 10 * 512 and np.array_equal(sf_from_atoms(buf, 300, 37), sf)
    offs = _sf_offsets(300, 37).ravel()
    assert np.unique(offs).size == offs.size  # a bijection onto its image


def _fp4_inputs(R, K, seed):
    g = np.random.default_rng(seed)
    a = (g.standard_normal((R, K)) * np.exp(g.uniform(-3, 3, (R, 1)))).astype(np.float32)
    a[:, g.choice(K, size=max(1, K // 100), replace=False)] *= 40
    if R > 2:
        a[1, :64] = 0.0                                   # all-zero blocks
        a[2, : K // 2] *= 1e-5                            # tiny blocks (E4M3 block scales near 0)
    return a.astype(np.float16)


@pytest.mark.parametrize("R,K", FP4_Q_SMALL)
def test_mxfp4_quantizer_bit_exact(wq, R, K):
    a = _fp4_inputs(R, K, seed=R * K + 5)
    q, s = wq.quantize_mxfp4(dev(a))
    torch.cuda.synchronize()
    rq, rs = oracle.quantize_mxfp4(a)
    assert host(s).size == wq.fp4_scale_bytes(R, K, False)
    assert np.array_equal(sf_from_atoms(host(s), R, K // 32), rs) and np.array_equal(host(q), rq)


@pytest.mark.parametrize("R,K", [rk for rk in FP4_Q_SMALL if rk[1] % 16 == 0])
def test_nvfp4_quantizer_bit_exact(wq, R, K):
    a = _fp4_inputs(R, K, seed=R * K + 6)
    q, s, t = wq.quantize_nvfp4(dev(a))
    torch.cuda.synchronize()
    rq, rs, rt = oracle.quantize_nvfp4(a)
    assert np.array_equal(host(t), rt)
    assert host(s).size == wq.fp4_scale_bytes(R, K, True)
    assert np.array_equal(sf_from_atoms(host(s), R, K // 16), rs) and np.array_equal(host(q), rq)


def test_fp4_quantizers_every_e2m1_midpoint(wq):
    # v / scale next to every E2M1 rounding boundary, both signs: the row maximum 6 fixes the
    # MX exponent at 0 (2^floor(log2 6) / 4 = 1) and the NV block scale at 1 x S
    vals = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float64)
    row = np.concatenate([vals, vals * (1 + 2 ** -9), vals * (1 - 2 ** -9), [6.0] * 11])
    a = np.stack([row[:32], -row[:32]]).astype(np.float16)
    q, s = wq.quantize_mxfp4(dev(a))
    rq, rs = oracle.quantize_mxfp4(a)
    assert np.array_equal(sf_from_atoms(host(s), 2, 1), rs) and np.array_equal(host(q), rq)
    q, s, t = wq.quantize_nvfp4(dev(a))
    rq, rs, rt = oracle.quantize_nvfp4(a)
    assert np.array_equal(host(t), rt) and np.array_equal(sf_from_atoms(host(s), 2, 2), rs)
    assert np.array_equal(host(q), rq)


FP4_GEMM_SMALL = [(1, 1, 256), (128, 128, 256), (130, 300, 512), (64, 40, 1024), (257, 513, 256),
                  (300, 1000, 2048), (512, 1024, 4096)]


@pytest.mark.parametrize("M,N,K", FP4_GEMM_SMALL)
@pytest.mark.parametrize("nv", [False, True])
def test_gemm_fp4_small(wq, M, N, K, nv):
    a = _fp4_inputs(M, K, seed=M + K)
    b = (_fp4_inputs(N, K, seed=N + 2 * K).astype(np.float32) * 0.05).astype(np.float16)
    if nv:
        qa, sa, ta = oracle.quantize_nvfp4(a)
        qb, sb, tb = oracle.quantize_nvfp4(b)
        y = wq.gemm_fp4(dev(qa), dev(sf_to_atoms(sa)), dev(qb), dev(sf_to_atoms(sb)), dev(ta), dev(tb))
        tav, tbv = float(ta[0]), float(tb[0])
    else:
        qa, sa = oracle.quantize_mxfp4(a)
        qb, sb = oracle.quantize_mxfp4(b)
        y = wq.gemm_fp4(dev(qa), dev(sf_to_atoms(sa)), dev(qb), dev(sf_to_atoms(sb)))
        tav = tbv = 1.0
    torch.cuda.synchronize()
    ms, ns = sample_rows(M, 64, seed=1), sample_rows(N, 96, seed=2)
    ry, rb = oracle.gemm_fp4_ref(nv, qa, sa, tav, qb, sb, tbv, K, ms, ns)
    assert_within_bound(host(y)[np.ix_(ms, ns)].astype(np.float64), ry, rb, f"fp4 nv={nv} M={M} N={N} K={K}")
    assert wq.device_status() == 0


@pytest.mark.parametrize("nv", [False, True])
def test_gemm_fp4_scale_factor_placement(wq, nv):
    # Every A row and every K block gets its own power-of-two scale (B all ones with scale 1): each
    # output is the sum of A's decoded row, so a misplaced factor (row, block or byte) shows up.
    # Scales 2^-3 .. 2^3 keep every partial sum a multiple of 2^-4 below 2^15: exact in fp32.
    M, N, K = 256, 128, 512
    bs = 16 if nv else 32
    g = np.random.default_rng(7)
    qa = g.integers(0, 256, (M, K // 2), dtype=np.uint8)
    qb = np.full((N, K // 2), 0x22, np.uint8)                       # E2M1 1.0 in both nibbles
    if nv:   # E4M3 codes of 2^e: exponent field e + 7, mantissa 0
        sa = ((g.integers(-3, 4, (M, K // bs)) + 7) << 3).astype(np.uint8)
        sb = np.full((N, K // bs), 7 << 3, np.uint8)                # 1.0
        one = np.ones(1, np.float32)
        y, acc = wq.gemm_fp4(dev(qa), dev(sf_to_atoms(sa)), dev(qb), dev(sf_to_atoms(sb)), dev(one), dev(one),
                             return_acc=True)
    else:
        sa = (g.integers(-3, 4, (M, K // bs)) + 127).astype(np.uint8)
        sb = np.full((N, K // bs), 127, np.uint8)
        y, acc = wq.gemm_fp4(dev(qa), dev(sf_to_atoms(sa)), dev(qb), dev(sf_to_atoms(sb)), return_acc=True)
    torch.cuda.synchronize()
    ry, _ = oracle.gemm_fp4_ref(nv, qa, sa, 1.0, qb, sb, 1.0, K)
    assert np.array_equal(host(acc).astype(np.float64), ry)


def test_fp4_w4a4_full_size(wq):
    # The W8A8 layer's shapes (X [2048, 8192], W [8192, 8192]) in MXFP4 and NVFP4, quantized on the
    # GPU and multiplied on the tensor cores; codes and scales checked on sampled rows.
    M, N, K = 2048, 8192, 8192
    X = workloads.config_activations("w8a8_smoothquant", M, K)
    W = workloads.config_weight("w8a8_smoothquant")
    ms, ns = sample_rows(M, 48, seed=8), sample_rows(N, 64, seed=9)
    xa, wa = dev(X), dev(W)
    for nv in (False, True):
        if nv:
            qx, sx, tx = wq.quantize_nvfp4(xa)
            qw, sw, tw = wq.quantize_nvfp4(wa)
            y = wq.gemm_fp4(qx, sx, qw, sw, tx, tw)
            rqx, rsx, rtx = oracle.quantize_nvfp4(X)
            assert np.array_equal(host(tx), rtx)
            tv = (float(host(tx)[0]), float(host(tw)[0]))
        else:
            qx, sx = wq.quantize_mxfp4(xa)
            qw, sw = wq.quantize_mxfp4(wa)
            y = wq.gemm_fp4(qx, sx, qw, sw)
            rqx, rsx = oracle.quantize_mxfp4(X[ms])
            tv = (1.0, 1.0)
        torch.cuda.synchronize()
        F = K // (16 if nv else 32)
        hqx, hqw = host(qx), host(qw)
        hsx, hsw = sf_from_atoms(host(sx), M, F), sf_from_atoms(host(sw), N, F)
        assert np.array_equal(hqx[ms], rqx[ms] if nv else rqx) and np.array_equal(hsx[ms], rsx[ms] if nv else rsx)
        ry, rb = oracle.gemm_fp4_ref(nv, hqx, hsx, tv[0], hqw, hsw, tv[1], K, ms, ns)
        assert_within_bound(host(y)[np.ix_(ms, ns)].astype(np.float64), ry, rb, f"fp4 full nv={nv}")
    assert wq.device_status() == 0


# --------------------------------------------------------------------------
# Split last round of the persistent W8A8 / FP8 GEMMs: 160 tiles of 128 x 256 on 148 SMs leave 12
# tiles after one whole round; CTA pairs share them (half of K each, summed through distributed
# shared memory).  Every output of those tiles (n-tiles 14 and 15) is checked, plus a sample.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("fp8", [False, True])
def test_w8a8_split_last_round(wq, fp8):
    M, N, K = 1280, 4096, 512
    g = np.random.default_rng(17 + fp8)
    sx = (g.random(M, dtype=np.float32) + 0.01) * 0.05
    sw = (g.random(N, dtype=np.float32) + 0.01) * 0.01
    ns = np.arange(14 * 256, 16 * 256, dtype=np.int32)
    ms = np.arange(M, dtype=np.int32)
    if fp8:
        xq, wq8 = _random_e4m3(g, (M, K)), _random_e4m3(g, (N, K))
        y, acc = wq.gemm_fp8(dev(xq), dev(sx), dev(wq8), dev(sw), return_acc=True)
        torch.cuda.synchronize()
        ry, rb = oracle.gemm_fp8_ref(xq, sx, wq8, sw, ms, ns)
    else:
        xq = g.integers(-128, 128, (M, K), dtype=np.int8)
        wq8 = g.integers(-128, 128, (N, K), dtype=np.int8)
        y, acc = wq.gemm_w8a8(dev(xq), dev(sx), dev(wq8), dev(sw), return_acc=True)
        torch.cuda.synchronize()
        racc, ry, rb = oracle.gemm_w8a8_ref(xq, sx, wq8, sw, ms, ns)
        assert np.array_equal(host(acc)[:, ns].astype(np.int64), racc)
    assert_within_bound(host(y)[:, ns].astype(np.float64), ry, rb, f"split round fp8={fp8}")
    ms2, ns2 = sample_rows(M, 64, seed=3), sample_rows(N, 64, seed=4)
    if fp8:
        ry2, rb2 = oracle.gemm_fp8_ref(xq, sx, wq8, sw, ms2, ns2)
    else:
        _, ry2, rb2 = oracle.gemm_w8a8_ref(xq, sx, wq8, sw, ms2, ns2)
    assert_within_bound(host(y)[np.ix_(ms2, ns2)].astype(np.float64), ry2, rb2, f"split round sample fp8={fp8}")
    assert wq.device_status() == 0


# --------------------------------------------------------------------------
# GPTQ and AWQ on the GPU (fp32) against the fp64 oracle: the Hessian and the
# factor within rounding, GPTQ with U = I exactly round-to-nearest, GPTQ's
# objective and codes close to the oracle's and below RTN, AWQ's choice,
# scales and codes exact
# --------------------------------------------------------------------------
def _calib_inputs(seed, N=256, K=512, T=512, outliers=()):
    g = np.random.default_rng(seed)
    x = g.standard_normal((T, K)).astype(np.float32)
    x += 0.8 * (g.standard_normal((T, 4)) @ g.standard_normal((4, K))).astype(np.float32)
    for c in outliers:
        x[:, c] *= 30.0
    w = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    return x.astype(np.float16), w.astype(np.float16)


def _cal_objective(x, w, qw, sc, qz, K, s=None):
    what = oracle.dequant_int4(qw, sc, qz, K, 128)
    if s is not None:
        what = what / s.astype(np.float64)[None, :]
    d = w.astype(np.float64) - what
    return float(np.sum((x.astype(np.float64) @ d.T) ** 2))


def test_hessian_and_gptq_factor(wq):
    x, _ = _calib_inputs(61, K=256, T=300)
    H = wq.hessian(dev(x))
    U = wq.gptq_prepare(H, 0.01)
    torch.cuda.synchronize()
    rH = oracle.hessian(x)
    assert np.max(np.abs(host(H) - rH)) <= 1e-5 * np.max(np.abs(rH))
    rU = oracle.gptq_hinv_chol(rH, 0.01)
    hU = host(U).astype(np.float64)
    assert np.allclose(np.triu(hU), hU)
    assert np.linalg.norm(hU - rU) <= 1e-3 * np.linalg.norm(rU)


def test_gptq_with_identity_factor_is_round_to_nearest(wq):
    _, w = _calib_inputs(62)
    K = w.shape[1]
    qw, sc, qz = wq.gptq_quantize(dev(w), torch.eye(K, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    rqw, rsc, rqz = oracle.quantize_group_int4(w, 128)
    assert np.array_equal(host(qw, np.uint32), rqw) and np.array_equal(host(qz, np.uint32), rqz)
    assert np.array_equal(host(sc).view(np.uint16), rsc.view(np.uint16))


def test_gptq_matches_the_oracle_objective(wq):
    x, w = _calib_inputs(63)
    K = w.shape[1]
    U = wq.gptq_prepare(wq.hessian(dev(x)), 0.01)
    qw, sc, qz = wq.gptq_quantize(dev(w), U)
    torch.cuda.synchronize()
    rU = oracle.gptq_hinv_chol(oracle.hessian(x), 0.01)
    rqw, rsc, rqz = oracle.gptq(w, rU, 128)
    hqw, hsc, hqz = host(qw, np.uint32), host(sc), host(qz, np.uint32)
    e_gpu = _cal_objective(x, w, hqw, hsc, hqz, K)
    e_ref = _cal_objective(x, w, rqw, rsc, rqz, K)
    tqw, tsc, tqz = oracle.quantize_group_int4(w, 128)
    e_rtn = _cal_objective(x, w, tqw, tsc, tqz, K)
    assert abs(e_gpu - e_ref) <= 0.02 * e_ref and e_gpu < 0.8 * e_rtn
    codes_gpu, codes_ref = oracle.unpack_int4_codes(hqw, K), oracle.unpack_int4_codes(rqw, K)
    assert np.mean(codes_gpu == codes_ref) >= 0.97
    assert np.mean(hsc.view(np.uint16) == rsc.view(np.uint16)) >= 0.95


def test_awq_matches_the_oracle(wq):
    x, w = _calib_inputs(64, outliers=(3, 70, 200, 301))
    K = w.shape[1]
    qw, sc, qz, s, err, best = wq.awq(dev(w), dev(x))
    torch.cuda.synchronize()
    rqw, rsc, rqz, rs, rbest, rerr = oracle.awq(w, x, oracle.hessian(x), 128)
    assert int(host(best)[0]) == rbest
    assert np.allclose(host(err), rerr, rtol=1e-4)
    assert np.array_equal(host(s), rs)
    assert np.array_equal(host(qw, np.uint32), rqw) and np.array_equal(host(qz, np.uint32), rqz)
    assert np.array_equal(host(sc).view(np.uint16), rsc.view(np.uint16))
    assert rbest > 0 and rerr[rbest] < rerr[0]


# --------------------------------------------------------------------------
# bf16 activations: the W4A16 GEMV (any group size) and GEMM (tensor cores with bf16 tiles)
# against the oracle with bf16 x; bf16 outputs, so the bound is 2^-8 sum |w^ x| + 1e-5
# (bf16 rounding of the output and, in the GEMM, of each dequantized weight)
# --------------------------------------------------------------------------
BF16_RTOL = 2.0 ** -8

BF16_CASES = [  # (kind, M, N, K, g)
    ("gemv", 1, 300, 1024, 128), ("gemv", 8, 520, 2048, 32), ("gemv", 5, 129, 768, 64), ("gemv", 3, 77, 512, 256),
    ("gemm", 16, 300, 1024, 128), ("gemm", 64, 1000, 4096, 128), ("gemm", 100, 384, 3072, 64),
    ("gemm", 12, 300, 1280, 128), ("gemm", 130, 260, 2048, 32), ("gemm", 48, 640, 16384, 256),
]


@pytest.mark.parametrize("kind,M,N,K,g", BF16_CASES)
def test_w4a16_bf16_activations(wq, kind, M, N, K, g):
    w = _special_weights(N, K, seed=M + N + K + 7)
    rqw, rsc, rqz = oracle.quantize_group_int4(w, g)
    x = workloads.activations(M, K, 0.01, 50.0, seed=M + 1, tensor_id=N).astype(np.float32)
    xt = torch.from_numpy(x).to(torch.bfloat16)
    xbits = xt.view(torch.int16).numpy().view(np.uint16)
    f = wq.gemv_w4a16_bf16 if kind == "gemv" else wq.gemm_w4a16_bf16
    y = f(xt.cuda(), dev(rqw.view(np.int32)), dev(rsc), dev(rqz.view(np.int32)), g)
    torch.cuda.synchronize()
    rows = sample_rows(N, 300, seed=K)
    y_ref, bound = oracle.matmul_w4a16_ref_bf16(xbits, rqw, rsc, rqz, K, g, rows=rows)
    hy = y.float().cpu().numpy().astype(np.float64)[:, rows]
    err = np.abs(hy - y_ref)
    lim = BF16_RTOL * bound + ATOL
    assert not (err > lim).any(), f"bf16 {kind} M={M} N={N} K={K} g={g}: worst excess {(err - lim).max():.3e}"
    assert wq.device_status() == 0
