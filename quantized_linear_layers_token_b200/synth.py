"""Seeded synthetic workloads.

This module only draws random numbers and names shapes.  It holds none of the
layer's arithmetic, so both the CUDA path and the CPU oracle can be fed from
it.  Every draw uses numpy's PCG64 with ``seed = 1000 + workload index`` and
an independent sub-stream per (shape, draw) from ``SeedSequence.spawn``.

Workloads (shapes follow the models the pages evaluate: LLaMA-2 7B / 70B
linears in the QQQ review, Phi-3-mini linears in the Quaff notes):

* ``small``     single 512x512 W4A8 per-channel linear, M = 16, 2% outlier
                channels scaled by U[50, 100], gamma = 0.9, one step.
* ``llama7b_w4_decode``   7B layer set, W4A8 per-channel, M in {1, 4, 16, 64},
                1% outlier channels x100.
* ``llama7b_w4g128_prefill``  same layer set, W4A8 g128, M in {512, 2048,
                4096}; 0.1% of weight entries scaled x20.
* ``phi3_w8_quaff``  Phi-3-mini linears, W8A8, M = 4096, 2/5/5/8% outlier
                channels (qkv / o / gate_up / down) with magnitudes U[50,100]
                drifting by U[0.8, 1.2] per step, X redrawn each step, 20 steps.
* ``llama70b_w4g128``  70B layer set, W4A8 g128, M in {1, 16, 128, 1024, 8192},
                1% outlier channels x100, W ~ N(0, 0.015).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

W4_PERCHANNEL = 0
W4_G128 = 1
W8_PERCHANNEL = 2

LLAMA7B_SHAPES = [  # (name, K, N)
    ("q_proj", 4096, 4096), ("k_proj", 4096, 4096), ("v_proj", 4096, 4096),
    ("o_proj", 4096, 4096), ("gate_proj", 4096, 11008), ("up_proj", 4096, 11008),
    ("down_proj", 11008, 4096),
]
PHI3_SHAPES = [
    ("qkv_proj", 3072, 9216), ("o_proj", 3072, 3072), ("gate_up_proj", 3072, 16384),
    ("down_proj", 8192, 3072),
]
PHI3_OUTLIER_FRAC = {"qkv_proj": 0.02, "o_proj": 0.05, "gate_up_proj": 0.05, "down_proj": 0.08}
LLAMA70B_SHAPES = [
    ("q_proj", 8192, 8192), ("kv_proj", 8192, 1024), ("up_proj", 8192, 28672),
    ("down_proj", 28672, 8192),
]


@dataclass
class Workload:
    name: str
    index: int
    fmt: int
    shapes: list
    ms: list
    outlier_frac: dict | float
    x_mult: tuple  # ("uniform", lo, hi) or ("const", v)
    w_std: float
    w_spike_frac: float = 0.0
    w_spike_mult: float = 1.0
    gamma: float = 0.9
    steps: int = 1
    drift: tuple | None = None
    extra: dict = field(default_factory=dict)

    def n_outliers(self, name: str, K: int) -> int:
        f = self.outlier_frac[name] if isinstance(self.outlier_frac, dict) else self.outlier_frac
        return int(round(f * K))


WORKLOADS = {
    "small": Workload("small", 0, W4_PERCHANNEL, [("linear", 512, 512)], [16], 0.02,
                      ("uniform", 50.0, 100.0), 0.02),
    "llama7b_w4_decode": Workload("llama7b_w4_decode", 1, W4_PERCHANNEL, LLAMA7B_SHAPES,
                                  [1, 4, 16, 64], 0.01, ("const", 100.0), 0.02),
    "llama7b_w4g128_prefill": Workload("llama7b_w4g128_prefill", 2, W4_G128, LLAMA7B_SHAPES,
                                       [512, 2048, 4096], 0.01, ("const", 100.0), 0.02,
                                       w_spike_frac=0.001, w_spike_mult=20.0),
    "phi3_w8_quaff": Workload("phi3_w8_quaff", 3, W8_PERCHANNEL, PHI3_SHAPES, [4096],
                              PHI3_OUTLIER_FRAC, ("uniform", 50.0, 100.0), 0.02, steps=20,
                              drift=(0.8, 1.2)),
    "llama70b_w4g128": Workload("llama70b_w4g128", 4, W4_G128, LLAMA70B_SHAPES,
                                [1, 16, 128, 1024, 8192], 0.01, ("const", 100.0), 0.015),
}


def rng_for(index: int, *path: int) -> np.random.Generator:
    """PCG64 stream for workload ``index``; ``path`` selects a spawned
    sub-stream (e.g. shape number, then draw kind)."""
    ss = np.random.SeedSequence(1000 + index)
    for p in path:
        ss = ss.spawn(p + 1)[p]
    return np.random.Generator(np.random.PCG64(ss))


def outlier_channels(rng: np.random.Generator, K: int, n: int) -> np.ndarray:
    """``n`` distinct sorted channel indices in [0, K)."""
    if n <= 0:
        return np.zeros(0, np.int32)
    return np.sort(rng.choice(K, size=n, replace=False)).astype(np.int32)


def channel_multipliers(rng: np.random.Generator, n: int, spec: tuple) -> np.ndarray:
    if spec[0] == "const":
        return np.full(n, spec[1], np.float32)
    return rng.uniform(spec[1], spec[2], size=n).astype(np.float32)


def activations(rng: np.random.Generator, M: int, K: int, O: np.ndarray,
                mult: np.ndarray) -> np.ndarray:
    """X fp16 [M][K]: N(0, 1) with the channels in ``O`` multiplied by ``mult``."""
    x = rng.standard_normal((M, K), dtype=np.float32)
    if len(O):
        x[:, O] *= mult[None, :]
    return x.astype(np.float16)


def weights(rng: np.random.Generator, K: int, N: int, std: float, spike_frac: float = 0.0,
            spike_mult: float = 1.0) -> np.ndarray:
    """W fp16 [K][N] ~ N(0, std^2), with ``spike_frac`` of the entries (seeded
    positions) multiplied by ``spike_mult``."""
    w = rng.standard_normal((K, N), dtype=np.float32) * np.float32(std)
    if spike_frac > 0:
        n = int(round(spike_frac * K * N))
        idx = rng.choice(K * N, size=n, replace=False)
        w.reshape(-1)[idx] *= np.float32(spike_mult)
    return w.astype(np.float16)


def offq_signs(seed: int = 0) -> np.ndarray:
    """Signs d (int8 [128]) of the partially random Hadamard matrix D H of
    the OffQ transform: d_0 = +1 (so the matrix's first row is all ones),
    the other 127 seeded +-1 (draw kind 7)."""
    d = np.where(rng_for(5, seed, 7).random(128) < 0.5, -1, 1).astype(np.int8)
    d[0] = 1
    return d


def offq_activations(M: int, K: int, seed: int = 0, outlier_mult: tuple = (20.0, 60.0)) -> np.ndarray:
    """X fp16 [M][K] for the OffQ layer: N(0, 1), with the first channel of
    every 128-channel group scaled by U[20, 60] per group -- the layout the
    offline top-1 PCA rotation leaves (each group's outlier energy in its
    first channel)."""
    rng = rng_for(5, seed, 8, M % 997)
    x = rng.standard_normal((M, K), dtype=np.float32)
    mult = rng.uniform(outlier_mult[0], outlier_mult[1], size=K // 128).astype(np.float32)
    x[:, 0::128] *= mult[None, :]
    return x.astype(np.float16)


def offq_weights(K: int, N: int, seed: int = 0, std: float = 0.02) -> np.ndarray:
    """W fp16 [K][N] for the OffQ layer: N(0, std^2) i.i.d. (draw kind 9)."""
    rng = rng_for(5, seed, 9, N % 997)
    return (rng.standard_normal((K, N), dtype=np.float32) * np.float32(std)).astype(np.float16)


def grad_output(index: int, shape_idx: int, M: int, N: int, std: float = 2.0 ** -7) -> np.ndarray:
    """Upstream gradient dY (fp16 [M][N]) for the input-gradient path:
    N(0, std^2) i.i.d., a stand-in for the gradient a fine-tuning loss sends
    back through the layer (draw kind 5 of the shape's sub-streams)."""
    rng = rng_for(index, shape_idx, 5, M % 997)
    return (rng.standard_normal((M, N), dtype=np.float32) * np.float32(std)).astype(np.float16)


def outlier_scales(index: int, shape_idx: int, n: int, lo: float = 1.0, hi: float = 8.0) -> np.ndarray:
    """Scales s (fp32 [n]) a forward pass left on the outlier channels: U[lo, hi]
    (draw kind 6)."""
    return rng_for(index, shape_idx, 6).uniform(lo, hi, size=n).astype(np.float32)


def layer(workload: str | Workload, shape_idx: int, M: int | None = None, step: int = 0,
          K: int | None = None, N: int | None = None, n_outliers: int | None = None,
          with_weights: bool = True) -> dict:
    """Draw one layer of a workload: X (fp16 [M][K]), W (fp16 [K][N]), O.

    ``K``, ``N``, ``n_outliers`` override the workload's shape (used for
    small parity cases drawn with the same distributions).  ``step`` > 0
    redraws X and applies the per-step outlier drift (the Phi-3 workload)."""
    wl = WORKLOADS[workload] if isinstance(workload, str) else workload
    name, K0, N0 = wl.shapes[shape_idx]
    K = K0 if K is None else K
    N = N0 if N is None else N
    M = wl.ms[0] if M is None else M
    nO = wl.n_outliers(name, K) if n_outliers is None else n_outliers
    O = outlier_channels(rng_for(wl.index, shape_idx, 0), K, nO)
    mult = channel_multipliers(rng_for(wl.index, shape_idx, 1), len(O), wl.x_mult)
    if wl.drift is not None and step > 0:
        drng = rng_for(wl.index, shape_idx, 2)
        for _ in range(step):
            mult = (mult * drng.uniform(wl.drift[0], wl.drift[1], size=len(O))).astype(np.float32)
    X = activations(rng_for(wl.index, shape_idx, 3, step, M % 997), M, K, O, mult)
    out = {"name": name, "K": K, "N": N, "M": M, "O": O, "X": X, "fmt": wl.fmt,
           "gamma": wl.gamma}
    if with_weights:
        out["W"] = weights(rng_for(wl.index, shape_idx, 4), K, N, wl.w_std, wl.w_spike_frac,
                           wl.w_spike_mult)
    return out
