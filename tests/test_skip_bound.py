"""The skip rule of the screened passes, checked in float64 on the CPU (no GPU, no kernel):
on a clustered problem at the oracle's potentials, a key tile (256 points) or a 16-point
group inside a kept tile is left out of a 64-row block when, for every row i of the block,
Hmax - kappa dist(x_i, box)^2 < thr_i, with thr_i = max_j z_ij - (24 + log2 M). Whatever is
left out of a row's sum must then be below 2^-24 of that sum (each left-out term is below
2^-(24 + log2 M) of the row's largest term, and there are at most M of them). The kernels
use a lower bound on max_j z_ij, which lowers thr_i and only leaves out less."""
import math

import numpy as np
import pytest

import oracle
from streaming_sinkhorn_b200 import workloads


def morton_order(p, lo, hi, bits=10):
    q = np.clip(((p - lo) / (hi - lo) * ((1 << bits) - 1)).astype(np.int64), 0, (1 << bits) - 1)
    code = np.zeros(len(p), dtype=np.int64)
    for bit in range(bits):
        for k in range(p.shape[1]):
            code |= ((q[:, k] >> bit) & 1) << (p.shape[1] * bit + k)
    return np.argsort(code, kind="stable")


def box_skip(xb, thr, kappa, lo, hi, hmax):
    """True when no row of the block (rows xb, thresholds thr) may need the set of keys with
    bounding box [lo, hi] and largest bias hmax."""
    gap = np.maximum(np.maximum(lo[None, :] - xb, xb - hi[None, :]), 0.0)
    return bool(np.all(hmax - kappa * (gap * gap).sum(1) < thr))


@pytest.mark.parametrize("seed,eps", [(0, None), (1, 2.0 ** (-40.0 / 3.0))],
                         ids=["eps-spacing-rule", "eps-of-2^20-points"])
def test_left_out_mass_is_below_2_pow_minus_24(seed, eps):
    w = workloads.clustered_cube(n=2048, seed=40 + seed, n_iters=6, eps=eps)
    f, g = oracle.potentials(w.x, w.y, w.a, w.b, w.eps, w.n_iters)
    x, y = w.x.astype(np.float64), w.y.astype(np.float64)
    lo = np.minimum(x.min(0), y.min(0))
    hi = np.maximum(x.max(0), y.max(0))
    ox, oy = morton_order(x, lo, hi), morton_order(y, lo, hi)
    xs, ys = x[ox], y[oy]
    kappa = math.log2(math.e) / w.eps
    h = kappa * g[oy] + np.log2(w.b[oy].astype(np.float64))  # key biases, sorted order
    z = h[None, :] - kappa * ((xs[:, None, :] - ys[None, :, :]) ** 2).sum(-1)
    margin = 24.0 + math.log2(len(ys))
    thr = z.max(1) - margin
    kept = np.ones(z.shape, dtype=bool)
    tiles = groups = 0
    for r0 in range(0, len(xs), 64):
        rb = slice(r0, r0 + 64)
        for t0 in range(0, len(ys), 256):
            tk = slice(t0, t0 + 256)
            if box_skip(xs[rb], thr[rb], kappa, ys[tk].min(0), ys[tk].max(0), h[tk].max()):
                kept[rb, tk] = False
                tiles += 1
                continue
            for g0 in range(t0, min(t0 + 256, len(ys)), 16):
                gk = slice(g0, g0 + 16)
                if box_skip(xs[rb], thr[rb], kappa, ys[gk].min(0), ys[gk].max(0), h[gk].max()):
                    kept[rb, gk] = False
                    groups += 1
    # the rule leaves out tiles and groups on this problem ...
    assert tiles > 0 and groups > 0 and kept.mean() < 0.9
    # ... and every row loses less than 2^-24 of its sum (relative to the row's largest term)
    e = np.exp2(z - z.max(1, keepdims=True))
    left_out = np.where(kept, 0.0, e).sum(1)
    assert np.all(left_out <= 2.0 ** -24 * e.sum(1))
    # each left-out term is below 2^-margin of its row's largest
    assert np.all(np.where(kept, -np.inf, z - z.max(1, keepdims=True)) < -margin)
