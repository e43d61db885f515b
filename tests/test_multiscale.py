"""The coarse-to-fine solve on the GPU: it reaches the same converged solution as the
oracle (up to the potentials' gauge constant), and on a clustered problem the coarse stage
saves fine iterations against a solve from g = 0."""
import numpy as np
import pytest

import oracle
import streaming_sinkhorn_b200 as fs
from streaming_sinkhorn_b200 import workloads
from tests.parity_util import inputs

pytestmark = pytest.mark.gpu


def test_multiscale_reaches_the_oracle_solution():
    w = workloads.random_small(2000, 2500, 2, seed=41, eps=0.2, n_iters=10)
    x, y, a, b = inputs(w)
    tol = 1e-7
    f, g, rep = fs.solve_multiscale(x, y, a, b, eps=w.eps, cell_points=16, coarse_iters=10,
                                    max_rounds=6,
                                    stop_mode="marginal", stop_tol=tol, stop_check_every=5,
                                    stop_max_iter=5000)
    assert rep["rounds"] >= 1 and rep["fine"]["converged"] is True
    fr, gr, *_ = oracle.solve(w.x, w.y, w.a, w.b, w.eps, stop_mode="marginal", stop_tol=1e-10,
                              stop_check_every=10, stop_max_iter=100000)
    df = f.cpu().numpy().astype(np.float64) - fr
    dg = g.cpu().numpy().astype(np.float64) - gr
    # the same potentials up to (f + c, g - c)
    assert np.ptp(df) < 2e-3 and np.ptp(dg) < 2e-3, (np.ptp(df), np.ptp(dg))
    assert abs(df.mean() + dg.mean()) < 2e-3
    c = fs.cost(x, y, f, g, a, b, eps=w.eps).item()
    assert c == pytest.approx(oracle.cost(w.x, w.y, w.a, w.b, w.eps, fr, gr), rel=1e-4)


def test_coarse_stage_saves_fine_iterations():
    w = workloads.clustered_cube(n=32768, seed=42, n_iters=10, eps=3e-4)
    x, y, a, b = inputs(w)
    tol = 0.05 / w.n  # a marginal violation of 5 % of a point's mass
    kw = dict(stop_mode="marginal", stop_tol=tol, stop_check_every=5, stop_max_iter=2000)
    _, _, plain = fs.solve(x, y, a, b, eps=w.eps, **kw)
    f, g, rep = fs.solve_multiscale(x, y, a, b, eps=w.eps, cell_points=8, coarse_iters=50,
                                    max_rounds=10, lift_tol=tol, **kw)
    assert plain["converged"] is True and rep["fine"]["converged"] is True
    assert rep["fine"]["iters_run"] < plain["iters_run"], (rep, plain)
    res = fs.marginal_residual(x, y, f, g, a, b, eps=w.eps).cpu().numpy()
    assert max(res[1], res[3]) <= tol
