"""Seeded synthetic inputs for the SVG-EAR attention hot path.

This module is shared by the CUDA path, the CPU oracle and the benchmark.  It
holds NO arithmetic of the method itself: it only draws random token matrices
shaped like the video-DiT attention layers that SVG-EAR targets, rounds them
to the working dtype, and picks the seeded k-means initial rows.

Workloads (SVG-EAR, §5 "Models"): Wan2.2 produces 21 frames x 3,600 tokens =
75,600 tokens; HunyuanVideo 33 x 3,600 = 118,800 tokens.  The real activations
and the VBench / Penguin prompt sets are not available, so these generators
stand in for them.

Recipe (one reading, written down because the workload text leaves it open):

* Every (config, head, stream) draws from its own numpy
  ``Generator(PCG64(SeedSequence([cfg_seed, head, stream])))`` with
  ``cfg_seed = 1000 + config number`` and streams Q=0, K=1, V=2,
  Q-init=3, K-init=4, mixture-labels=5.
* Token t has ONE mixture component z_t shared by Q, K and V (stream 5).
  Each of Q, K, V has its own centres mu ~ N(0, I_d).  Noise eps ~ N(0, I_d).
* Mixture configs: x_t = mu_{z_t} + sigma * eps_t.
* Grid configs: x_t = F_t + mu_{z_t} + sigma * eps_t where F is an i.i.d.
  N(0,1) field over the (frames, height, width) latent grid, blurred by a
  separable Gaussian (std 2 cells, radius 6, half-sample-symmetric
  "reflect" borders) and rescaled to unit std per channel.  Tokens are in
  raster order, frame-major.
* Values are drawn in fp64 and rounded (round-to-nearest-even) to the config
  dtype; every consumer reads the rounded values.
* k-means init: C distinct token rows drawn with ``rng.choice(N, C,
  replace=False)`` (kept in drawn order) from the rounded matrix.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor
from typing import Optional, Sequence

import numpy as np

STREAM_Q, STREAM_K, STREAM_V, STREAM_QINIT, STREAM_KINIT, STREAM_Z = 0, 1, 2, 3, 4, 5


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic attention layer: shapes, generator recipe and EAR hyper-parameters."""
    name: str
    number: int                 # config number; cfg_seed = 1000 + number
    heads: int                  # batch x heads (batch is 1 everywhere)
    n: int                      # tokens (N_q = N_k)
    d: int
    dtype: str                  # "f32" or "bf16"
    n_centres: int
    sigma: float
    c_q: int
    c_k: int
    iters: int
    density: float
    grid: Optional[tuple] = None      # (frames, height, width) for field configs
    label_mode: str = "uniform"       # "balanced" | "uniform" | "zipf"
    zipf_s: float = 1.2

    @property
    def cfg_seed(self) -> int:
        return 1000 + self.number

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


TINY = Workload("tiny-1head-N1024-d64-f32", 1, heads=1, n=1024, d=64, dtype="f32",
                n_centres=16, sigma=0.3, c_q=16, c_k=16, iters=10, density=0.25,
                label_mode="balanced")
MID = Workload("mid-8head-N8192-d128-bf16", 2, heads=8, n=8192, d=128, dtype="bf16",
               n_centres=64, sigma=0.4, c_q=64, c_k=128, iters=8, density=0.15)
WAN = Workload("wan2.x-layer-40head-N75600-d128-bf16", 3, heads=40, n=75600, d=128,
               dtype="bf16", n_centres=200, sigma=0.5, c_q=100, c_k=500, iters=5,
               density=0.10, grid=(21, 45, 80))
HUNYUAN = Workload("hunyuanvideo-layer-24head-N118800-d128-bf16", 4, heads=24, n=118800,
                   d=128, dtype="bf16", n_centres=300, sigma=0.5, c_q=100, c_k=500,
                   iters=5, density=0.10, grid=(33, 45, 80))
SKEW = Workload("wan2.x-zipf1.2-40head-N75600-d128-bf16", 5, heads=40, n=75600, d=128,
                dtype="bf16", n_centres=200, sigma=0.5, c_q=100, c_k=500, iters=5,
                density=0.10, grid=(21, 45, 80), label_mode="zipf")
SKEW_DENSITIES = (0.05, 0.10, 0.20, 0.40, 1.0)

CONFIGS = {1: TINY, 2: MID, 3: WAN, 4: HUNYUAN, 5: SKEW}


def _rng(cfg_seed: int, head: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([cfg_seed, head, stream])))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even to bfloat16; returns float32 holding bf16-exact values."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).reshape(f.shape)


def bf16_bits(x_bf16_exact: np.ndarray) -> np.ndarray:
    """uint16 bit pattern of float32 values that are already bf16-exact."""
    return (np.ascontiguousarray(x_bf16_exact, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return round_to_bf16(x)
    raise ValueError(f"unknown dtype {dtype!r}")


def mixture_labels(w: Workload, head: int, n: Optional[int] = None) -> np.ndarray:
    n = w.n if n is None else n
    rng = _rng(w.cfg_seed, head, STREAM_Z)
    if w.label_mode == "balanced":
        if n % w.n_centres:
            raise ValueError("balanced labels need n divisible by n_centres")
        return rng.permutation(np.repeat(np.arange(w.n_centres), n // w.n_centres))
    if w.label_mode == "uniform":
        return rng.integers(0, w.n_centres, size=n)
    if w.label_mode == "zipf":
        k = np.arange(1, w.n_centres + 1, dtype=np.float64)
        p = k ** (-w.zipf_s)
        return rng.choice(w.n_centres, size=n, p=p / p.sum())
    raise ValueError(w.label_mode)


def _smoothed_field(rng: np.random.Generator, grid: tuple, d: int) -> np.ndarray:
    from scipy.ndimage import gaussian_filter1d
    f = rng.standard_normal((*grid, d), dtype=np.float64).astype(np.float32)
    for axis in range(3):
        f = gaussian_filter1d(f, sigma=2.0, axis=axis, mode="reflect", truncate=3.0)
    f = f.reshape(-1, d)
    f -= f.mean(axis=0, keepdims=True)
    f /= f.std(axis=0, keepdims=True)
    return f


def token_matrix(w: Workload, head: int, stream: int, z: np.ndarray) -> np.ndarray:
    """One head's Q (stream 0), K (1) or V (2) as float32 holding dtype-exact values."""
    rng = _rng(w.cfg_seed, head, stream)
    n = z.shape[0]
    mu = rng.standard_normal((w.n_centres, w.d))
    x = np.empty((n, w.d), dtype=np.float64)
    if w.grid is not None:
        if int(np.prod(w.grid)) != n:
            raise ValueError("grid does not match token count")
        x[:] = _smoothed_field(rng, w.grid, w.d)
    else:
        x[:] = 0.0
    x += mu[z]
    x += w.sigma * rng.standard_normal((n, w.d))
    return round_to_dtype(x, w.dtype)


def init_rows(w: Workload, head: int, stream: int, x: np.ndarray, c: int) -> np.ndarray:
    """Seeded k-means init: c distinct rows of the rounded matrix x, in drawn order."""
    rng = _rng(w.cfg_seed, head, stream)
    idx = rng.choice(x.shape[0], size=c, replace=False)
    return np.ascontiguousarray(x[idx], dtype=np.float32)


@dataclasses.dataclass
class LayerInputs:
    """Per-layer inputs, float32 arrays holding dtype-exact values, shape [BH, N, d]."""
    workload: Workload
    heads: Sequence[int]
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    q_init: np.ndarray   # [BH, C_q, d] float32
    k_init: np.ndarray   # [BH, C_k, d] float32


def make_head(w: Workload, head: int):
    z = mixture_labels(w, head)
    q = token_matrix(w, head, STREAM_Q, z)
    k = token_matrix(w, head, STREAM_K, z)
    v = token_matrix(w, head, STREAM_V, z)
    qi = init_rows(w, head, STREAM_QINIT, q, w.c_q)
    ki = init_rows(w, head, STREAM_KINIT, k, w.c_k)
    return q, k, v, qi, ki


def make_layer(w: Workload, heads: Optional[Sequence[int]] = None, threads: int = 8) -> LayerInputs:
    heads = list(range(w.heads)) if heads is None else list(heads)
    bh = len(heads)
    q = np.empty((bh, w.n, w.d), np.float32)
    k = np.empty_like(q)
    v = np.empty_like(q)
    qi = np.empty((bh, w.c_q, w.d), np.float32)
    ki = np.empty((bh, w.c_k, w.d), np.float32)

    def one(slot):
        q[slot], k[slot], v[slot], qi[slot], ki[slot] = make_head(w, heads[slot])

    if threads > 1 and bh > 1:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(one, range(bh)))
    else:
        for s in range(bh):
            one(s)
    return LayerInputs(w, heads, q, k, v, qi, ki)
