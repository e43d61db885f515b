"""The coarse-to-fine solve on the GPU: it reaches the same converged solution as the
oracle (up to the potentials' gauge constant), and on a clustered problem the coarse stage
saves fine iterations against a solve from g = 0."""
import numpy as np
import pytest

import oracle
import streaming_sinkhorn_b200 as fs
from streaming_sinkhorn_b200 import workloads
from tests.parity_util import assert_potential_close, inputs

pytestmark = pytest.mark.gpu


def test_multiscale_reaches_the_oracle_solution():
    """The coarse stage only initialises the fine solve, so its result is the same fixed
    point as a plain solve (FlashSinkhorn 2 abstract): after removing the gauge constant c
    of (f + c, g - c), f and g must meet the potential bar 1e-4 max(1, |f_ref|).

    Bound of the stopping error: a solve stopped at a marginal violation v (largest
    |P1 - a|, |P^T 1 - b| entry) leaves each row or column mass off by at most v, which is a
    relative error v / min(a) of that row's sum, i.e. eps * v / min(a) in its potential
    (f_i = -eps LSE + ...), and the next update carries it to the other side once more:
    |f - c - f*|, |g + c - g*| <= 2 eps v / min(a, b). At eps = 0.2, v = 1e-8 and
    min(a, b) ~ 2.5e-4 that is 1.6e-5, well inside the 1e-4 bar; the oracle is solved to
    1e-10, a hundred times tighter still.
    """
    w = workloads.random_small(2000, 2500, 2, seed=41, eps=0.2, n_iters=10)
    x, y, a, b = inputs(w)
    tol = 1e-8
    f, g, rep = fs.solve_multiscale(x, y, a, b, eps=w.eps, cell_points=16, coarse_iters=10,
                                    max_rounds=6,
                                    stop_mode="marginal", stop_tol=tol, stop_check_every=5,
                                    stop_max_iter=10000)
    assert rep["rounds"] >= 1 and rep["fine"]["converged"] is True, rep
    fr, gr, *_ = oracle.solve(w.x, w.y, w.a, w.b, w.eps, stop_mode="marginal", stop_tol=1e-10,
                              stop_check_every=10, stop_max_iter=100000)
    wmin = min(float(w.a[w.a > 0].min()), float(w.b[w.b > 0].min()))
    assert 2.0 * w.eps * tol / wmin < 0.25e-4  # the stopping error is far below the bar
    fn = f.cpu().numpy().astype(np.float64)
    gn = g.cpu().numpy().astype(np.float64)
    c = 0.5 * ((fn - fr).mean() - (gn - gr).mean())  # the gauge constant
    assert_potential_close(fn - c, fr, "f")
    assert_potential_close(gn + c, gr, "g")
    cost = fs.cost(x, y, f, g, a, b, eps=w.eps).item()
    assert cost == pytest.approx(oracle.cost(w.x, w.y, w.a, w.b, w.eps, fr, gr), rel=1e-4)


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
