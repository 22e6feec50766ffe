"""Seeded synthetic inputs shaped like the source pages' workloads.

This module holds random number draws only: no scale, zero point, rounding or
matmul arithmetic of the method lives here.  Both the CUDA path's tests and
benchmark and the CPU oracle take their inputs from it; nothing else is shared
between the two.

The pages measure on real checkpoints (Qwen3-0.6B, Qwen2.5-0.5B) and real text,
none of which exist here; these generators stand in for them with the same
shapes and the same structure (bell-shaped weights, a few large outlier
weights, activation channels tens of times larger than the rest).

Every tensor has its own stream: ``numpy.random.Generator(PCG64(SeedSequence(
[seed, tensor_id])))``.  Normals are drawn in float32 and rounded once to the
storage dtype (round-to-nearest-even via numpy's fp16 conversion).
"""
from __future__ import annotations

import dataclasses

import numpy as np

__all__ = ["CONFIGS", "Config", "rng", "weight_normal", "weight_lognormal_rows",
           "weight_every_nth_outlier", "activations", "w8a8_activations", "config_inputs"]


def rng(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(tensor_id)])))


def _normal(g: np.random.Generator, shape, sigma) -> np.ndarray:
    out = g.standard_normal(shape, dtype=np.float32)
    out *= np.float32(sigma) if np.isscalar(sigma) else np.asarray(sigma, np.float32)
    return out


def weight_normal(N: int, K: int, sigma: float, seed: int, tensor_id: int = 0,
                  dtype=np.float16) -> np.ndarray:
    """W[n, k] ~ N(0, sigma), [N out, K in] row-major (nn.Linear layout)."""
    return _normal(rng(seed, tensor_id), (N, K), sigma).astype(dtype)


def weight_every_nth_outlier(N: int, K: int, sigma: float, nth: int, mult: float, seed: int,
                             tensor_id: int = 0, dtype=np.float32) -> np.ndarray:
    """N(0, sigma) with every nth element (flat index i, (i+1) % nth == 0) times mult."""
    w = _normal(rng(seed, tensor_id), (N, K), sigma).reshape(-1)
    w[nth - 1::nth] *= np.float32(mult)
    return w.reshape(N, K).astype(dtype)


def weight_lognormal_rows(N: int, K: int, seed: int, tensor_id: int = 0, log_mu=np.log(0.02),
                          log_sigma=0.5, p_outlier=0.001, outlier_mult=30.0,
                          dtype=np.float16) -> np.ndarray:
    """Row scales sigma_n = exp(N(log_mu, log_sigma)); entries N(0, sigma_n); each entry is
    multiplied by outlier_mult with probability p_outlier."""
    g = rng(seed, tensor_id)
    sig = np.exp(g.normal(log_mu, log_sigma, size=(N, 1))).astype(np.float32)
    w = g.standard_normal((N, K), dtype=np.float32) * sig
    mask = g.random((N, K), dtype=np.float32) < np.float32(p_outlier)
    w[mask] *= np.float32(outlier_mult)
    return w.astype(dtype)


def activations(B: int, K: int, outlier_frac: float, outlier_mult: float, seed: int,
                tensor_id: int = 100, dtype=np.float16) -> np.ndarray:
    """x[b, k] ~ N(0, 1); floor(outlier_frac * K) channels (sampled without replacement,
    the same channels for every row) are multiplied by outlier_mult."""
    g = rng(seed, tensor_id)
    x = g.standard_normal((B, K), dtype=np.float32)
    n_out = int(np.floor(outlier_frac * K))
    if n_out:
        ch = g.choice(K, size=n_out, replace=False)
        x[:, ch] *= np.float32(outlier_mult)
    return x.astype(dtype)


def w8a8_activations(M: int, K: int, n_outlier: int = 64, mult: float = 60.0, seed: int = 5,
                     tensor_id: int = 200) -> np.ndarray:
    """X ~ N(0,1) [M, K] fp16 with n_outlier fixed channels (drawn once from seed) x mult."""
    ch = rng(seed, 0).choice(K, size=n_outlier, replace=False)
    x = rng(seed, tensor_id).standard_normal((M, K), dtype=np.float32)
    x[:, ch] *= np.float32(mult)
    return x.astype(np.float16)


@dataclasses.dataclass(frozen=True)
class Config:
    """One workload: W4A16 weight shapes [(N, K), ...] and batches, or a W8A8 problem."""
    name: str
    seed: int
    shapes: tuple          # ((N, K), ...) weight matrices [out, in]
    batches: tuple         # activation batch sizes for the W4A16 matmuls
    description: str


CONFIGS = {
    "tiny_w4a16": Config("tiny_w4a16", 0, ((256, 512),), (1,),
              "fp32 W 256x512 N(0,0.02), every 97th element x20; x fp16 [1,512] N(0,1)"),
    "decode_4096": Config("decode_4096", 2, ((4096, 4096),), (1, 4),
              "fp16 W 4096x4096, row sigma lognormal(ln 0.02, 0.5), 0.1% entries x30; "
              "x N(0,1) with 1% of channels x50"),
    "mlp_8b": Config("mlp_8b", 3, ((14336, 4096), (4096, 14336)), (1, 8, 16),
              "fp16 W N(0,0.02) gate/up 14336x4096 and down 4096x14336; x with 1% channels x50; "
              "also INT8 per-channel (W8A16) on the same weights"),
    "llama70b_class": Config("llama70b_class", 4, ((28672, 8192), (8192, 28672)), (1, 16, 64),
              "fp16 W N(0,0.015) 28672x8192 and 8192x28672; x with 0.5% channels x100"),
    "w8a8_smoothquant": Config("w8a8_smoothquant", 5, ((8192, 8192),), (2048,),
              "X fp16 [2048, 8192] N(0,1) with 64 fixed channels x60; W fp16 8192x8192 N(0,0.02); "
              "alpha 0.5"),
}

_X_OUTLIERS = {"tiny_w4a16": (0.0, 1.0), "decode_4096": (0.01, 50.0), "mlp_8b": (0.01, 50.0),
               "llama70b_class": (0.005, 100.0)}
_W_SIGMA = {"mlp_8b": 0.02, "llama70b_class": 0.015}


def config_weight(cfg: str, shape_index: int = 0, shape=None) -> np.ndarray:
    """The weight matrix of workload `cfg` (a key of CONFIGS), optionally at another [N, K]."""
    c = CONFIGS[cfg]
    N, K = shape if shape is not None else c.shapes[shape_index]
    if cfg == "tiny_w4a16":
        return weight_every_nth_outlier(N, K, 0.02, 97, 20.0, c.seed, shape_index, np.float32)
    if cfg == "decode_4096":
        return weight_lognormal_rows(N, K, c.seed, shape_index)
    if cfg in ("mlp_8b", "llama70b_class"):
        return weight_normal(N, K, _W_SIGMA[cfg], c.seed, shape_index)
    if cfg == "w8a8_smoothquant":
        return weight_normal(N, K, 0.02, c.seed, 1)
    raise KeyError(cfg)


def config_activations(cfg: str, B: int, K: int, tensor_id: int = 100) -> np.ndarray:
    """Activation rows [B, K] of workload `cfg` (a key of CONFIGS)."""
    c = CONFIGS[cfg]
    if cfg == "w8a8_smoothquant":
        return w8a8_activations(B, K, seed=c.seed)
    frac, mult = _X_OUTLIERS[cfg]
    return activations(B, K, frac, mult, c.seed, tensor_id + B)


def config_inputs(cfg: str):
    """All tensors of a config: {"weights": [W...], "x": {B: [x per weight]}}."""
    c = CONFIGS[cfg]
    ws = [config_weight(cfg, i) for i in range(len(c.shapes))]
    xs = {B: [config_activations(cfg, B, K) for (_, K) in c.shapes] for B in c.batches}
    return {"weights": ws, "x": xs}
