"""Write the oracle's outputs for the named configurations to ``tests/golden/``.

Calls only the fp64 oracle (``oracle/``) and the seeded input generators; no value
here comes from the CUDA path. Usage::

    python tests/golden/make_golden.py 0 1 2      # configurations by 0-based index

Besides the five configurations, ``extra`` problems (by name) are written the same way:
``cluster_32k_d3`` is the 2^20-point clustered recipe (1000 Gaussians of std 0.01 in the
unit cube, clipped) at 2^15 points with the same eps = 2^(-40/3) and 20 iterations, small
enough for the oracle to run in full (2.7e10 pair evaluations)::

    python tests/golden/make_golden.py cluster_32k_d3

Each file ``<config name>.npz`` holds: the SHA-256 of the fp32 inputs it was computed
from, eps and the iteration count, the potentials f and g after the fixed iteration
count (alternating schedule, g starting at zero), the dual objective at (f, g), the
envelope gradient (all rows, or a seeded sample of rows for d > 16), and the four
marginal-residual norms [L1 row, Linf row, L1 col, Linf col].
"""
import dataclasses
import hashlib
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from streaming_sinkhorn_b200 import workloads  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))


def input_digest(w) -> str:
    h = hashlib.sha256()
    for arr in (w.x, w.y, w.a, w.b):
        h.update(np.ascontiguousarray(arr, np.float32).tobytes())
    return h.hexdigest()


EXTRA = {
    "cluster_32k_d3": lambda: workloads.clustered_cube(n=1 << 15, d=3, k=1000, std=0.01, seed=4,
                                                       eps=2.0 ** (-40.0 / 3.0), n_iters=20),
}


def grad_rows(w, extra: bool = False) -> np.ndarray:
    """All rows for the configurations with d <= 16; a seeded sample of 512 rows for d > 16
    and for the extra problems."""
    if w.d <= 16 and not extra:
        return np.arange(w.n, dtype=np.int64)
    rng = np.random.default_rng(12345)
    return np.sort(rng.choice(w.n, size=512, replace=False)).astype(np.int64)


def make(i) -> str:
    if isinstance(i, str):
        w = dataclasses.replace(EXTRA[i](), name=i)
    else:
        w = workloads.config(i)
    t0 = time.time()
    f, g = oracle.potentials(w.x, w.y, w.a, w.b, w.eps, w.n_iters)
    t1 = time.time()
    c = oracle.cost(w.x, w.y, w.a, w.b, w.eps, f, g)
    rows = grad_rows(w, extra=isinstance(i, str))
    gr = oracle.grad_x(w.x, w.y, w.a, w.b, w.eps, g, rows=rows)
    res = oracle.marginal_residual(w.x, w.y, w.a, w.b, w.eps, f, g)
    t2 = time.time()
    path = os.path.join(HERE, f"{w.name}.npz")
    np.savez_compressed(path, digest=np.array(input_digest(w)), eps=np.float64(w.eps),
                        n_iters=np.int64(w.n_iters), f=f, g=g, cost=np.float64(c),
                        grad_rows=rows, grad=gr, residual=res,
                        oracle_seconds=np.float64(t1 - t0), threads=np.int64(oracle.threads()))
    print(f"{w.name}: potentials {t1 - t0:.1f}s, rest {t2 - t1:.1f}s, cost {c!r}, "
          f"residual {res}", flush=True)
    return path


if __name__ == "__main__":
    for arg in sys.argv[1:]:
        make(arg if arg in EXTRA else int(arg))
