"""Seeded synthetic point clouds shaped like the workloads on the pages.

This module draws inputs only. It holds none of the transport arithmetic, so the
CUDA path and the fp64 oracle can both consume exactly the same fp32 arrays.

Shapes follow the pages' workload grids: the usage examples of the SinkSLOT README
("Basic Usage", N=10000, d=2, eps=0.05, 200 iterations; "Gradient Flow", N=1000 with
the target shifted by +3), its "Reproducing the paper" grid (d=3 and d=64 Gaussian
families, N up to 50k), and the FlashSinkhorn 2 abstract's large N-body-scale solve
(blur equal to the mean interparticle distance). No public dataset is read.

Every array is drawn with ``numpy.random.default_rng(seed)`` in float64 in the
order written in each recipe, then cast once to float32. Weight vectors are
returned explicitly even where they are uniform.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic entropic-OT problem instance (inputs only)."""

    name: str
    x: np.ndarray  # (N, d) float32
    y: np.ndarray  # (M, d) float32
    a: np.ndarray  # (N,) float32, nonnegative
    b: np.ndarray  # (M,) float32, nonnegative
    eps: float
    n_iters: int
    seed: int

    @property
    def n(self) -> int:
        return int(self.x.shape[0])

    @property
    def m(self) -> int:
        return int(self.y.shape[0])

    @property
    def d(self) -> int:
        return int(self.x.shape[1])


def _f32(v: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(v, dtype=np.float32)


def _uniform(k: int) -> np.ndarray:
    return np.full((k,), 1.0 / k, dtype=np.float64)


def gaussian_shifted(n: int = 1000, d: int = 2, shift: float = 3.0, seed: int = 0,
                     eps: float = 0.05, n_iters: int = 100) -> Workload:
    """x ~ N(0, I_d); y ~ N(0, I_d) with ``shift`` added to coordinate 0; uniform weights.

    Draw order: x, then y.
    """
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, d))
    y = rng.standard_normal((n, d))
    y[:, 0] += shift
    return Workload("gaussian_shifted", _f32(x), _f32(y), _f32(_uniform(n)), _f32(_uniform(n)),
                    eps, n_iters, seed)


def gaussian_pair(n: int = 10000, m: int | None = None, d: int = 2, seed: int = 1,
                  eps: float = 0.05, n_iters: int = 200) -> Workload:
    """x, y ~ N(0, I_d) drawn independently; uniform weights. Draw order: x, then y."""
    m = n if m is None else m
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, d))
    y = rng.standard_normal((m, d))
    return Workload("gaussian_pair", _f32(x), _f32(y), _f32(_uniform(n)), _f32(_uniform(m)),
                    eps, n_iters, seed)


def cube_to_mixture(n: int = 20000, m: int = 30000, d: int = 3, k: int = 8, std: float = 0.05,
                    seed: int = 2, eps: float = 0.01, n_iters: int = 200) -> Workload:
    """x ~ U[0,1]^d; y = 8-component Gaussian mixture (means ~ U[0,1]^d, std 0.05).

    Weights a_i, b_j ~ U[0.5, 1.5], each divided by its float64 sum.
    Draw order: x, means, y labels, y noise, a, b.
    """
    rng = np.random.default_rng(seed)
    x = rng.random((n, d))
    means = rng.random((k, d))
    labels = rng.integers(0, k, size=m)
    y = means[labels] + std * rng.standard_normal((m, d))
    a = rng.uniform(0.5, 1.5, size=n)
    b = rng.uniform(0.5, 1.5, size=m)
    a = a / a.sum()
    b = b / b.sum()
    return Workload("cube_to_mixture", _f32(x), _f32(y), _f32(a), _f32(b), eps, n_iters, seed)


def mixture_pair(n: int = 50000, m: int | None = None, d: int = 64, k: int = 10,
                 mean_scale: float = 2.0, std: float = 1.0, seed: int = 3, eps: float = 1.0,
                 n_iters: int = 100, clip_unit_cube: bool = False) -> Workload:
    """x, y drawn independently from one k-component Gaussian mixture.

    Means = mean_scale * N(0, I_d) when ``clip_unit_cube`` is False, otherwise
    means ~ U[0,1]^d and points are clipped to [0,1]^d. Equal component
    probabilities; per-dimension std ``std``; uniform weights.
    Draw order: means, x labels, x noise, y labels, y noise.
    """
    m = n if m is None else m
    rng = np.random.default_rng(seed)
    if clip_unit_cube:
        means = rng.random((k, d))
    else:
        means = mean_scale * rng.standard_normal((k, d))
    lx = rng.integers(0, k, size=n)
    x = means[lx] + std * rng.standard_normal((n, d))
    ly = rng.integers(0, k, size=m)
    y = means[ly] + std * rng.standard_normal((m, d))
    if clip_unit_cube:
        np.clip(x, 0.0, 1.0, out=x)
        np.clip(y, 0.0, 1.0, out=y)
    return Workload("mixture_pair", _f32(x), _f32(y), _f32(_uniform(n)), _f32(_uniform(m)),
                    eps, n_iters, seed)


def clustered_cube(n: int = 1 << 20, d: int = 3, k: int = 1000, std: float = 0.01, seed: int = 4,
                   eps: float | None = None, n_iters: int = 20) -> Workload:
    """Clustered unit-cube clouds: 1000 Gaussians (means ~ U[0,1]^3, std 0.01), clipped.

    eps defaults to (n^(-1/d))^2, the squared mean interparticle spacing of n points in
    the unit cube (the blur rule of the FlashSinkhorn 2 abstract).
    """
    if eps is None:
        eps = float(n) ** (-2.0 / d)
    w = mixture_pair(n=n, m=n, d=d, k=k, std=std, seed=seed, eps=eps, n_iters=n_iters,
                     clip_unit_cube=True)
    return dataclasses.replace(w, name="clustered_cube")


# The five named configurations, in order.
CONFIG_NAMES = ("c1_gauss_shift_1k_d2", "c2_gauss_10k_d2", "c3_cube_mix_20k30k_d3",
                "c4_mix_50k_d64", "c5_cluster_1m_d3")


def config(i: int, seed_offset: int = 0) -> Workload:
    """Configuration ``i`` (0-based) of the five named workloads, at full size.

    ``seed_offset`` draws an independent instance of the same recipe (replicas of a
    multi-process run); 0 is the configuration itself.
    """
    o = seed_offset
    if i == 0:
        w = gaussian_shifted(n=1000, d=2, shift=3.0, seed=0 + o, eps=0.05, n_iters=100)
    elif i == 1:
        w = gaussian_pair(n=10000, d=2, seed=1 + o, eps=0.05, n_iters=200)
    elif i == 2:
        w = cube_to_mixture(n=20000, m=30000, d=3, k=8, std=0.05, seed=2 + o, eps=0.01,
                            n_iters=200)
    elif i == 3:
        w = mixture_pair(n=50000, d=64, k=10, mean_scale=2.0, std=1.0, seed=3 + o, eps=1.0,
                         n_iters=100)
    elif i == 4:
        w = clustered_cube(n=1 << 20, d=3, k=1000, std=0.01, seed=4 + o,
                           eps=2.0 ** (-40.0 / 3.0), n_iters=20)
    else:
        raise IndexError(f"no configuration {i}")
    return dataclasses.replace(w, name=CONFIG_NAMES[i])


def c5_eps() -> float:
    """eps of the 2^20-point clustered configuration: (2^(-20/3))^2 = 2^(-40/3)."""
    return 2.0 ** (-40.0 / 3.0)


def random_small(n: int, m: int, d: int, seed: int, eps: float = 0.5, zero_frac: float = 0.0,
                 mass: float = 1.0, n_iters: int = 10) -> Workload:
    """Small random problem for parity and edge-case tests.

    x ~ N(0, I), y ~ N(0, I) + 0.5; weights ~ U[0.5, 1.5] with a fraction ``zero_frac``
    set to zero (never all of them), both normalised to total ``mass``.
    Draw order: x, y, a, b, a-zero mask, b-zero mask.
    """
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, d))
    y = rng.standard_normal((m, d)) + 0.5
    a = rng.uniform(0.5, 1.5, size=n)
    b = rng.uniform(0.5, 1.5, size=m)
    za = rng.random(n) < zero_frac
    zb = rng.random(m) < zero_frac
    za[0] = False
    zb[0] = False
    a[za] = 0.0
    b[zb] = 0.0
    a = mass * a / a.sum()
    b = mass * b / b.sum()
    return Workload("random_small", _f32(x), _f32(y), _f32(a), _f32(b), eps, n_iters, seed)


def mean_spacing_eps(n: int, d: int) -> float:
    """(n^(-1/d))^2: squared mean spacing of n points in the unit cube."""
    return math.pow(float(n), -2.0 / d)
