"""GPU parity on small problems: the CUDA path (through the C ABI) against the fp64
oracle, element by element, on seeded inputs whose sizes span several tiles, ragged
tails, single points, zero weights and masses other than one."""
import numpy as np
import pytest

import oracle
import streaming_sinkhorn_b200 as fs
from streaming_sinkhorn_b200 import workloads
from tests.parity_util import (assert_cost_close, assert_grad_close, assert_potential_close,
                               dev, grad_rel, inputs, residual_tolerance)

pytestmark = pytest.mark.gpu

SHAPES = [  # (n, m, d, zero_frac, mass, eps)
    (1, 1, 2, 0.0, 1.0, 0.3),
    (2, 3, 3, 0.0, 1.0, 0.3),
    (31, 33, 3, 0.2, 1.0, 0.2),
    (64, 63, 2, 0.0, 2.5, 0.2),
    (127, 256, 3, 0.1, 1.0, 0.1),
    (257, 129, 1, 0.0, 1.0, 0.05),
    (1000, 999, 2, 0.05, 1.0, 0.05),
    (700, 1500, 3, 0.0, 0.4, 0.02),
    (300, 200, 4, 0.1, 1.0, 0.5),
    (129, 130, 5, 0.0, 1.0, 0.5),
    (200, 333, 8, 0.0, 1.0, 1.0),
    (150, 90, 16, 0.2, 1.0, 2.0),
    (100, 120, 17, 0.0, 1.0, 2.0),
    (96, 160, 32, 0.0, 1.0, 4.0),
    (130, 70, 64, 0.1, 1.0, 8.0),
    (96, 120, 96, 0.0, 1.0, 12.0),     # wide points: 64-coordinate K-chunks from here on
    (140, 130, 128, 0.1, 1.0, 16.0),
    (130, 100, 512, 0.0, 1.0, 64.0),
    (100, 90, 1024, 0.0, 1.0, 128.0),
]


def problem(n, m, d, zero_frac, mass, eps, seed=0, iters=7):
    return workloads.random_small(n, m, d, seed=seed + n + 7 * m + 31 * d, eps=eps,
                                  zero_frac=zero_frac, mass=mass, n_iters=iters)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "n{}-m{}-d{}".format(*s[:3]))
def test_potentials_cost_grad_residual(shape):
    w = problem(*shape)
    x, y, a, b = inputs(w)
    f, g = fs.potentials(x, y, a, b, eps=w.eps, n_iters=w.n_iters)
    fr, gr = oracle.potentials(w.x, w.y, w.a, w.b, w.eps, w.n_iters)
    assert_potential_close(f.cpu().numpy(), fr, "f")
    assert_potential_close(g.cpu().numpy(), gr, "g")

    c = fs.cost(x, y, f, g, a, b, eps=w.eps).item()
    # oracle cost at the GPU's own (f, g): checks the cost pass, not the iterate
    cr = oracle.cost(w.x, w.y, w.a, w.b, w.eps, f.cpu().numpy(), g.cpu().numpy())
    assert_cost_close(c, cr)
    assert_cost_close(c, oracle.cost(w.x, w.y, w.a, w.b, w.eps, fr, gr))

    gx = fs.grad_x(x, y, g, a, b, eps=w.eps).cpu().numpy()
    gxr = oracle.grad_x(w.x, w.y, w.a, w.b, w.eps, g.cpu().numpy())
    assert_grad_close(gx, gxr, rel=grad_rel(w.d))

    res, r, cc = fs.marginal_residual(x, y, f, g, a, b, eps=w.eps, marginals=True)
    fn, gn = f.cpu().numpy(), g.cpu().numpy()
    rr = oracle.plan_row_sums(w.x, w.y, w.a, w.b, w.eps, fn, gn)
    cr_ = oracle.plan_col_sums(w.x, w.y, w.a, w.b, w.eps, fn, gn)
    tol = residual_tolerance(w)
    np.testing.assert_allclose(r.cpu().numpy(), rr, rtol=1e-3, atol=tol)
    np.testing.assert_allclose(cc.cpu().numpy(), cr_, rtol=1e-3, atol=tol)
    resr = oracle.marginal_residual(w.x, w.y, w.a, w.b, w.eps, fn, gn)
    np.testing.assert_allclose(res.cpu().numpy(), resr, rtol=1e-3, atol=tol)


def test_single_pair_closed_form_on_gpu():
    x = dev(np.array([[0.3, -1.2, 2.0]], np.float32))
    y = dev(np.array([[1.1, 0.4, -0.5]], np.float32))
    C = float(((x - y) ** 2).sum())
    for wgt in (1.0, 0.25):
        a = dev(np.array([wgt], np.float32))
        f, g = fs.potentials(x, y, a, a, eps=0.7, n_iters=3)
        assert f.item() + g.item() == pytest.approx(C - 0.7 * np.log(wgt), rel=1e-5, abs=1e-5)


def test_uniform_weights_default():
    w = problem(300, 257, 2, 0.0, 1.0, 0.1)
    x, y, _, _ = inputs(w)
    f, g = fs.potentials(x, y, eps=w.eps, n_iters=5)
    u_a = np.full(w.n, 1.0 / w.n, np.float32)
    u_b = np.full(w.m, 1.0 / w.m, np.float32)
    fr, gr = oracle.potentials(w.x, w.y, u_a, u_b, w.eps, 5)
    assert_potential_close(f.cpu().numpy(), fr, "f")
    assert_potential_close(g.cpu().numpy(), gr, "g")


def test_warm_start_and_gauge():
    w = problem(200, 150, 3, 0.1, 1.0, 0.1)
    x, y, a, b = inputs(w)
    g0 = np.random.default_rng(5).standard_normal(w.m).astype(np.float32) * 0.2
    f, g = fs.potentials(x, y, a, b, eps=w.eps, n_iters=4, g_init=dev(g0))
    fr, gr = oracle.potentials(w.x, w.y, w.a, w.b, w.eps, 4, g_init=g0)
    assert_potential_close(f.cpu().numpy(), fr, "f")
    assert_potential_close(g.cpu().numpy(), gr, "g")
    # gauge: g0 - c gives (f + c, g - c)
    f2, g2 = fs.potentials(x, y, a, b, eps=w.eps, n_iters=4, g_init=dev(g0 - 0.5))
    np.testing.assert_allclose(f2.cpu().numpy(), f.cpu().numpy() + 0.5, atol=2e-5)
    np.testing.assert_allclose(g2.cpu().numpy(), g.cpu().numpy() - 0.5, atol=2e-5)


def test_column_residual_vanishes_after_g_update():
    w = problem(500, 700, 3, 0.0, 1.0, 0.05)
    x, y, a, b = inputs(w)
    f, g = fs.potentials(x, y, a, b, eps=w.eps, n_iters=3)
    res = fs.marginal_residual(x, y, f, g, a, b, eps=w.eps).cpu().numpy()
    assert res[3] < 1e-5 * b.max().item() + residual_tolerance(w)
    assert res[1] > 100 * res[3]


@pytest.mark.parametrize("case", ["mass", "negative", "nan_x", "nan_w", "zero_mass", "nan_g"])
def test_device_validation_errors(case):
    w = problem(50, 40, 2, 0.0, 1.0, 0.1)
    x, y, a, b = inputs(w)
    g0 = None
    if case == "mass":
        b = b * 1.01
    elif case == "negative":
        a = a.clone()
        a[3] = -1e-3
    elif case == "nan_x":
        x = x.clone()
        x[7, 1] = float("nan")
    elif case == "nan_w":
        b = b.clone()
        b[0] = float("inf")
    elif case == "zero_mass":
        a = a * 0
        b = b * 0
    elif case == "nan_g":
        g0 = y[:, 0].clone()
        g0[2] = float("nan")
    with pytest.raises(ValueError) as e:
        fs.potentials(x, y, a, b, eps=w.eps, n_iters=2, g_init=g0)
    expect = {"mass": "FS_ERR_MASS_MISMATCH", "negative": "FS_ERR_NEGATIVE_WEIGHT",
              "nan_x": "FS_ERR_NONFINITE_INPUT", "nan_w": "FS_ERR_NEGATIVE_WEIGHT",
              "zero_mass": "FS_ERR_ZERO_MASS", "nan_g": "FS_ERR_NONFINITE_INPUT"}[case]
    assert e.value.status == expect


def test_solve_host_matches_device_calls():
    w = problem(400, 333, 3, 0.0, 1.0, 0.05)
    out = fs.solve_host(w.x, w.y, w.a, w.b, eps=w.eps, n_iters=6)
    x, y, a, b = inputs(w)
    f, g = fs.potentials(x, y, a, b, eps=w.eps, n_iters=6)
    np.testing.assert_array_equal(out["f"].numpy(), f.cpu().numpy())
    np.testing.assert_array_equal(out["g"].numpy(), g.cpu().numpy())
    gx = fs.grad_x(x, y, g, a, b, eps=w.eps)
    np.testing.assert_array_equal(out["grad_x"].numpy(), gx.cpu().numpy())
    assert out["cost"][0].item() == pytest.approx(fs.cost(x, y, f, g, a, b, eps=w.eps).item(),
                                                 rel=1e-12)
    np.testing.assert_allclose(out["residual"].numpy(),
                               fs.marginal_residual(x, y, f, g, a, b, eps=w.eps).cpu().numpy(),
                               rtol=1e-12)


def test_repeated_calls_are_deterministic():
    w = problem(1000, 1000, 2, 0.0, 1.0, 0.05)
    x, y, a, b = inputs(w)
    f1, g1 = fs.potentials(x, y, a, b, eps=w.eps, n_iters=5)
    f2, g2 = fs.potentials(x, y, a, b, eps=w.eps, n_iters=5)
    assert bool((f1 == f2).all()) and bool((g1 == g2).all())


@pytest.mark.parametrize("n,m,launches", [
    (1000, 800, 1),    # at most 2^22 pairs: the whole solve in one cluster launch
    (3000, 2500, 8),   # above: one streaming pass per half-iteration
])
def test_kernel_timing_counts_launches(n, m, launches):
    w = problem(n, m, 3, 0.0, 1.0, 0.05)
    x, y, a, b = inputs(w)
    fs.timing_enable(True)
    fs.timing_reset()
    try:
        f, g = fs.potentials(x, y, a, b, eps=w.eps, n_iters=4)
        t = fs.timing_get()
    finally:
        fs.timing_enable(False)
    assert t["lse_pass"]["launches"] == launches
    assert t["lse_pass"]["pairs"] == pytest.approx(8 * n * m)
    assert t["lse_pass"]["total_ms"] > 0
    fr, gr = oracle.potentials(w.x, w.y, w.a, w.b, w.eps, 4)
    assert_potential_close(f.cpu().numpy(), fr, "f")
    assert_potential_close(g.cpu().numpy(), gr, "g")
