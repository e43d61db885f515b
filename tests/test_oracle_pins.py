"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these retypes the oracle's own formula: each compares it with a closed
form, an invariant, a different algorithm (Sinkhorn-Knopp scaling on an explicit
kernel matrix, Cuturi 2013, listed among the FS2 page's references), or a
numerical derivative. A plausible slip in ``oracle.c`` -- a dropped log-weight
term, a sign, a swapped operand, an off-by-one in the schedule -- fails one of them.
"""
import numpy as np
import pytest

import oracle
from streaming_sinkhorn_b200 import workloads


def dense_cost(x, y):
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    return ((x[:, None, :] - y[None, :, :]) ** 2).sum(-1)


def scaling_sinkhorn(x, y, a, b, eps, n_iters, g0=None):
    """Sinkhorn-Knopp on the explicit Gibbs kernel K = exp(-C/eps).

    u = a / (K v), v = b / (K^T u), v0 = b exp(g0/eps). Returns the potentials in the
    log-domain convention: f = -eps log(K v), g = -eps log(K^T u).
    """
    C = dense_cost(x, y)
    K = np.exp(-C / eps)
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    v = b.copy() if g0 is None else b * np.exp(np.asarray(g0, np.float64) / eps)
    for _ in range(n_iters):
        Kv = K @ v
        u = a / Kv
        Ktu = K.T @ u
        v = b / Ktu
    return -eps * np.log(Kv), -eps * np.log(Ktu)


def dense_plan(x, y, a, b, eps, f, g):
    C = dense_cost(x, y)
    return (np.asarray(a, np.float64)[:, None] * np.asarray(b, np.float64)[None, :]
            * np.exp((np.asarray(f)[:, None] + np.asarray(g)[None, :] - C) / eps))


def small(n, m, d, seed, eps=0.5, zero_frac=0.0, mass=1.0):
    w = workloads.random_small(n, m, d, seed, eps=eps, zero_frac=zero_frac, mass=mass)
    a = w.a.astype(np.float64)
    b = w.b.astype(np.float64)
    b *= a.sum() / b.sum()  # balance the masses exactly in float64
    return w.x.astype(np.float64), w.y.astype(np.float64), a, b, w.eps


# --- N = M = 1 -----------------------------------------------------------------------

@pytest.mark.parametrize("w", [1.0, 0.25, 3.0])
def test_single_pair_closed_form(w):
    """One point each, weights w: after one iteration f = C - eps log w, g = 0,
    so f + g = C - eps log w (= C for unit weights) and further iterations keep it."""
    x = np.array([[0.3, -1.2, 2.0]])
    y = np.array([[1.1, 0.4, -0.5]])
    C = float(((x - y) ** 2).sum())
    eps = 0.7
    a = np.array([w])
    b = np.array([w])
    for iters in (1, 2, 5):
        f, g = oracle.potentials(x, y, a, b, eps, iters)
        assert f[0] == pytest.approx(C - eps * np.log(w), rel=1e-14, abs=1e-14)
        assert g[0] == pytest.approx(0.0, abs=1e-13)
        assert f[0] + g[0] == pytest.approx(C - eps * np.log(w), rel=1e-14, abs=1e-14)


# --- brute-force scaling Sinkhorn ---------------------------------------------------------

@pytest.mark.parametrize("n,m,d,seed,zero_frac", [(7, 5, 2, 0, 0.0), (31, 40, 3, 1, 0.2),
                                                  (64, 33, 5, 2, 0.1), (1, 9, 2, 3, 0.0)])
@pytest.mark.parametrize("iters", [1, 2, 7])
def test_matches_scaling_sinkhorn(n, m, d, seed, zero_frac, iters):
    x, y, a, b, _ = small(n, m, d, seed, zero_frac=zero_frac)
    C = dense_cost(x, y)
    eps = float(C.max()) / 30.0  # keeps C/eps < 700 so exp(-C/eps) is finite
    f, g = oracle.potentials(x, y, a, b, eps, iters)
    fs, gs = scaling_sinkhorn(x, y, a, b, eps, iters)
    np.testing.assert_allclose(f, fs, rtol=1e-11, atol=1e-12 * C.max())
    np.testing.assert_allclose(g, gs, rtol=1e-11, atol=1e-12 * C.max())


def test_matches_scaling_with_warm_start():
    x, y, a, b, _ = small(20, 13, 3, 5)
    eps = float(dense_cost(x, y).max()) / 20.0
    g0 = np.random.default_rng(9).standard_normal(13) * 0.3
    f, g = oracle.potentials(x, y, a, b, eps, 4, g_init=g0)
    fs, gs = scaling_sinkhorn(x, y, a, b, eps, 4, g0=g0)
    np.testing.assert_allclose(f, fs, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(g, gs, rtol=1e-11, atol=1e-12)


def test_row_subset_equals_full_update():
    x, y, a, b, eps = small(50, 37, 3, 6)
    g = np.random.default_rng(1).standard_normal(37)
    full = oracle.lse_update(x, y, b, g, eps)
    rows = np.array([49, 0, 17, 17, 3])
    np.testing.assert_array_equal(oracle.lse_update(x, y, b, g, eps, rows=rows), full[rows])


# --- gauge invariance ---------------------------------------------------------------------

@pytest.mark.parametrize("c", [0.37, -2.5])
def test_gauge_shift(c):
    """Starting from g0 - c gives (f + c, g - c) at every iterate and the same cost."""
    x, y, a, b, eps = small(25, 18, 2, 7)
    f0, g0 = oracle.potentials(x, y, a, b, eps, 3)
    f1, g1 = oracle.potentials(x, y, a, b, eps, 3, g_init=np.full(18, -c))
    np.testing.assert_allclose(f1, f0 + c, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g1, g0 - c, rtol=0, atol=1e-12)
    assert oracle.cost(x, y, a, b, eps, f1, g1) == pytest.approx(
        oracle.cost(x, y, a, b, eps, f0, g0), rel=1e-12, abs=1e-12)


# --- marginals ----------------------------------------------------------------------------

def test_marginals_after_each_update():
    """Right after an f-update P 1 = a; right after a g-update P^T 1 = b (to rounding)."""
    x, y, a, b, eps = small(30, 22, 3, 8, zero_frac=0.2)
    f, g = oracle.potentials(x, y, a, b, eps, 2)
    r = oracle.plan_row_sums(x, y, a, b, eps, f, g)
    c = oracle.plan_col_sums(x, y, a, b, eps, f, g)
    np.testing.assert_allclose(c, b, rtol=1e-12, atol=1e-15)
    assert np.abs(r - a).max() > 1e-6  # not converged after 2 iterations
    f2 = oracle.lse_update(x, y, b, g, eps)  # fresh f-update
    np.testing.assert_allclose(oracle.plan_row_sums(x, y, a, b, eps, f2, g), a, rtol=1e-12,
                               atol=1e-15)


def test_marginals_at_convergence():
    x, y, a, b, _ = small(16, 12, 2, 9)
    eps = 1.0
    f, g = oracle.potentials(x, y, a, b, eps, 400)
    res = oracle.marginal_residual(x, y, a, b, eps, f, g)
    assert res[1] < 1e-13 and res[3] < 1e-13
    assert res[0] < 1e-12 and res[2] < 1e-12


def test_residual_matches_dense_plan():
    x, y, a, b, eps = small(19, 27, 3, 10, zero_frac=0.15)
    f, g = oracle.potentials(x, y, a, b, eps, 3)
    f = f + 0.01 * np.sin(np.arange(19))  # arbitrary (f, g), not an iterate
    P = dense_plan(x, y, a, b, eps, f, g)
    np.testing.assert_allclose(oracle.plan_row_sums(x, y, a, b, eps, f, g), P.sum(1), rtol=1e-13)
    np.testing.assert_allclose(oracle.plan_col_sums(x, y, a, b, eps, f, g), P.sum(0), rtol=1e-13)
    res = oracle.marginal_residual(x, y, a, b, eps, f, g)
    dr, dc = np.abs(P.sum(1) - a), np.abs(P.sum(0) - b)
    np.testing.assert_allclose(res, [dr.sum(), dr.max(), dc.sum(), dc.max()], rtol=1e-12)


# --- cost -----------------------------------------------------------------------------------

@pytest.mark.parametrize("mass", [1.0, 2.5, 0.3])
def test_cost_dual_objective(mass):
    """The explicit double sum equals the dense-plan dual objective, and right after a
    g-update (P^T 1 = b) it reduces to <f,a> + <g,b> - eps*m*(1 - m)."""
    x, y, a, b, eps = small(21, 14, 2, 11, mass=mass)
    f, g = oracle.potentials(x, y, a, b, eps, 3)
    P = dense_plan(x, y, a, b, eps, f, g)
    dense = f @ a + g @ b - eps * (P.sum() - a.sum() * b.sum())
    got = oracle.cost(x, y, a, b, eps, f, g)
    assert got == pytest.approx(dense, rel=1e-12, abs=1e-14)
    m = b.sum()
    assert got == pytest.approx(f @ a + g @ b - eps * m * (1.0 - m), rel=1e-10, abs=1e-12)


def test_large_eps_product_limit():
    """eps -> infinity: P -> a (x) b, so the cost tends to <C, a (x) b> (closed form in
    O(N + M)) with an error that shrinks like 1/eps, and the gradient tends to
    2 a_i (x_i - sum_j b_j y_j)."""
    x, y, a, b, _ = small(17, 23, 3, 12)
    a /= a.sum()  # unit mass exactly, so the -eps*m*(1-m) term vanishes
    b /= b.sum()
    C = dense_cost(x, y)
    closed = (a @ (x ** 2).sum(1)) + (b @ (y ** 2).sum(1)) - 2.0 * (a @ x) @ (b @ y)
    assert closed == pytest.approx(a @ C @ b, rel=1e-12)
    errs = []
    for scale in (1e3, 1e4):
        eps = scale * C.max()
        f, g = oracle.potentials(x, y, a, b, eps, 5)
        errs.append(abs(oracle.cost(x, y, a, b, eps, f, g) - closed))
        gr = oracle.grad_x(x, y, a, b, eps, g)
        lim = 2.0 * a[:, None] * (x - (b @ y)[None, :])
        np.testing.assert_allclose(gr, lim, rtol=0, atol=50.0 / scale * np.abs(lim).max())
    assert errs[0] < 1e-2 * C.max()
    assert errs[1] < errs[0] / 5.0  # O(1/eps)


# --- gradient -------------------------------------------------------------------------------

def test_grad_matches_dense_plan():
    x, y, a, b, eps = small(23, 31, 3, 13, zero_frac=0.1)
    f, g = oracle.potentials(x, y, a, b, eps, 4)
    C = dense_cost(x, y)
    ft = -eps * np.log(np.exp(-C / eps) @ (b * np.exp(g / eps)))
    P = dense_plan(x, y, a, b, eps, ft, g)
    ref = 2.0 * (a[:, None] * x - P @ y)
    got = oracle.grad_x(x, y, a, b, eps, g)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-13)
    rows = np.array([5, 0, 22])
    np.testing.assert_array_equal(oracle.grad_x(x, y, a, b, eps, g, rows=rows), got[rows])


def test_grad_central_finite_difference():
    """At convergence the envelope gradient is the derivative of the solved cost.

    float64, 6 random directions per point, central differences; each perturbed cost
    is re-solved to convergence (SinkSLOT README, "dropped-term finite difference").
    """
    x, y, a, b, _ = small(10, 9, 2, 14)
    eps = 0.8
    iters = 600

    def solved_cost(xx):
        f, g = oracle.potentials(xx, y, a, b, eps, iters)
        return oracle.cost(xx, y, a, b, eps, f, g), f, g

    _, f, g = solved_cost(x)
    assert oracle.marginal_residual(x, y, a, b, eps, f, g)[1] < 1e-14
    grad = oracle.grad_x(x, y, a, b, eps, g)
    rng = np.random.default_rng(0)
    h = 1e-5
    worst = 0.0
    for i in range(x.shape[0]):
        for _ in range(6):
            v = rng.standard_normal(x.shape[1])
            v /= np.linalg.norm(v)
            xp = x.copy()
            xm = x.copy()
            xp[i] += h * v
            xm[i] -= h * v
            fd = (solved_cost(xp)[0] - solved_cost(xm)[0]) / (2 * h)
            worst = max(worst, abs(fd - grad[i] @ v))
    assert worst < 1e-8 * max(1.0, np.abs(grad).max() * 100)


def test_grad_fd_gap_shrinks_with_residual():
    """Before convergence the envelope gradient misses a term that vanishes with the
    marginal residual (SinkSLOT README, "gradient term split")."""
    x, y, a, b, _ = small(8, 8, 2, 15)
    eps = 0.5
    v = np.zeros_like(x)
    v[3] = [0.6, 0.8]
    h = 1e-5
    gaps = []
    for iters in (16, 64, 128):
        def c(xx):
            f, g = oracle.potentials(xx, y, a, b, eps, iters)
            return oracle.cost(xx, y, a, b, eps, f, g)
        _, g = oracle.potentials(x, y, a, b, eps, iters)
        fd = (c(x + h * v) - c(x - h * v)) / (2 * h)
        gaps.append(abs(fd - (oracle.grad_x(x, y, a, b, eps, g) * v).sum()))
    assert gaps[2] < gaps[1] < gaps[0]
    assert gaps[2] < 1e-9


# --- errors ---------------------------------------------------------------------------------

def test_mass_mismatch_raises():
    x, y, a, b, eps = small(5, 6, 2, 16)
    with pytest.raises(oracle.OracleError) as e:
        oracle.potentials(x, y, a, b * 1.001, eps, 2)
    assert e.value.code == -2
    oracle.potentials(x, y, a, b * (1 + 1e-7), eps, 2)  # inside the 1e-5 relative band


def test_zero_mass_and_negative_weight_raise():
    x, y, a, b, eps = small(5, 6, 2, 17)
    with pytest.raises(oracle.OracleError):
        oracle.potentials(x, y, np.zeros(5), np.zeros(6), eps, 1)
    bad = a.copy()
    bad[1] = -0.1
    with pytest.raises(oracle.OracleError):
        oracle.potentials(x, y, bad, b, eps, 1)
    with pytest.raises(oracle.OracleError):
        oracle.potentials(x, y, a, b, 0.0, 1)
    with pytest.raises(oracle.OracleError):
        oracle.potentials(x, y, a, b, eps, 0)


# --- the general solve: symmetric variant and stop modes ---------------------------------

def jacobi_scaling(x, y, a, b, eps, n_iters, alpha, g0=None):
    """The symmetric (Jacobi) blend in multiplicative form on the explicit Gibbs kernel:
    with U = exp(f/eps), V = b exp(g/eps), both new values come from the old pair,
    U' = U^(1-alpha) (K V)^(-alpha) and exp(g'/eps) = exp(g/eps)^(1-alpha) (K^T (a U))^(-alpha),
    from f = 0. Returns the list of (f, g) after each iteration."""
    C = dense_cost(x, y)
    K = np.exp(-C / eps)
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    U = np.ones(len(a))
    E = np.ones(len(b)) if g0 is None else np.exp(np.asarray(g0, np.float64) / eps)
    out = []
    for _ in range(n_iters):
        KV = K @ (b * E)
        KtU = K.T @ (a * U)
        U, E = U ** (1.0 - alpha) * KV ** (-alpha), E ** (1.0 - alpha) * KtU ** (-alpha)
        out.append((eps * np.log(U), eps * np.log(E)))
    return out


def dense_violation(x, y, a, b, eps, f, g):
    P = dense_plan(x, y, a, b, eps, f, g)
    return max(np.abs(P.sum(1) - a).max(), np.abs(P.sum(0) - b).max())


@pytest.mark.parametrize("alpha", [0.3, 0.5, 1.0])
@pytest.mark.parametrize("n,m,d,seed", [(7, 5, 2, 0), (40, 33, 3, 1)])
def test_symmetric_matches_jacobi_scaling(alpha, n, m, d, seed):
    x, y, a, b, _ = small(n, m, d, seed)
    eps = float(dense_cost(x, y).max()) / 25.0
    ref = jacobi_scaling(x, y, a, b, eps, 6, alpha)
    for iters in (1, 2, 6):
        f, g, it, conv, viol = oracle.solve(x, y, a, b, eps, n_iters=iters, variant="symmetric",
                                            alpha=alpha)
        assert it == iters and conv is None and np.isnan(viol)
        np.testing.assert_allclose(f, ref[iters - 1][0], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(g, ref[iters - 1][1], rtol=1e-11, atol=1e-12)


def test_symmetric_and_alternating_share_the_fixed_point():
    """Both schedules converge to the unique optimal plan (the potentials may differ by a
    constant (f + c, g - c), which leaves the plan and the cost unchanged)."""
    x, y, a, b, _ = small(30, 24, 2, 4)
    eps = float(dense_cost(x, y).max()) / 15.0
    fa, ga, *_ = oracle.solve(x, y, a, b, eps, n_iters=400)
    fs_, gs_, *_ = oracle.solve(x, y, a, b, eps, n_iters=1500, variant="symmetric", alpha=0.5)
    Pa = dense_plan(x, y, a, b, eps, fa, ga)
    Ps = dense_plan(x, y, a, b, eps, fs_, gs_)
    np.testing.assert_allclose(Ps, Pa, rtol=1e-7, atol=1e-12)
    shift = fs_ - fa
    assert np.ptp(shift) < 1e-7 and np.abs((gs_ - ga) + shift.mean()).max() < 1e-7


@pytest.mark.parametrize("variant", ["alternating", "symmetric"])
def test_marginal_stop_is_the_first_passing_check(variant):
    x, y, a, b, _ = small(25, 31, 2, 7)
    eps = float(dense_cost(x, y).max()) / 20.0
    tol, every = 1e-7, 4
    f, g, it, conv, viol = oracle.solve(x, y, a, b, eps, variant=variant, stop_mode="marginal",
                                        stop_tol=tol, stop_check_every=every, stop_max_iter=5000)
    assert conv is True and it % every == 0 and viol <= tol
    assert viol == pytest.approx(dense_violation(x, y, a, b, eps, f, g), rel=1e-9, abs=1e-15)
    # the check before it did not pass: rerun that many iterations with the fixed schedule
    if variant == "alternating":
        fp, gp = scaling_sinkhorn(x, y, a, b, eps, it - every)
    else:
        fp, gp = jacobi_scaling(x, y, a, b, eps, it - every, 0.5)[-1]
    assert dense_violation(x, y, a, b, eps, fp, gp) > tol


def test_potential_stop_measures_change_since_last_check():
    x, y, a, b, _ = small(20, 18, 3, 8)
    eps = float(dense_cost(x, y).max()) / 20.0
    tol, every = 1e-9, 3
    f, g, it, conv, viol = oracle.solve(x, y, a, b, eps, variant="symmetric", alpha=0.5,
                                        stop_mode="potential", stop_tol=tol,
                                        stop_check_every=every, stop_max_iter=5000)
    traj = jacobi_scaling(x, y, a, b, eps, it, 0.5)
    assert conv is True and it % every == 0 and viol < tol
    f0, g0 = traj[it - every - 1]
    expect = max(np.abs(traj[-1][0] - f0).max(), np.abs(traj[-1][1] - g0).max())
    assert viol == pytest.approx(expect, rel=1e-6, abs=1e-14)
    f1, g1 = traj[it - 2 * every - 1]
    assert max(np.abs(f0 - f1).max(), np.abs(g0 - g1).max()) >= tol


def test_stop_cap_reports_the_last_check():
    """A tolerance no check can meet: converged is False, iters_run is the cap, and the
    last check (after the capped iteration, 10 is not a multiple of 4) is reported."""
    x, y, a, b, _ = small(12, 9, 2, 9)
    eps = float(dense_cost(x, y).max()) / 10.0
    f, g, it, conv, viol = oracle.solve(x, y, a, b, eps, stop_mode="marginal", stop_tol=0.0,
                                        stop_check_every=4, stop_max_iter=10)
    assert conv is False and it == 10
    fs, gs = scaling_sinkhorn(x, y, a, b, eps, 10)
    np.testing.assert_allclose(f, fs, rtol=1e-11, atol=1e-12)
    assert viol == pytest.approx(dense_violation(x, y, a, b, eps, f, g), rel=1e-9, abs=1e-15)


def test_solve_argument_errors():
    x, y, a, b, eps = small(5, 6, 2, 10)
    for kw in ({"n_iters": 0}, {"variant": "symmetric", "alpha": 0.0},
               {"variant": "symmetric", "alpha": 1.5}, {"stop_mode": "marginal", "stop_max_iter": 0},
               {"stop_mode": "potential", "stop_check_every": 0},
               {"stop_mode": "marginal", "stop_tol": -1.0}):
        with pytest.raises(oracle.OracleError):
            oracle.solve(x, y, a, b, eps, **kw)


# --- transport products and the Hessian-vector product -----------------------------------

def converged(x, y, a, b, eps):
    f, g, it, conv, viol = oracle.solve(x, y, a, b, eps, stop_mode="marginal", stop_tol=1e-13,
                                        stop_check_every=10, stop_max_iter=20000)
    assert conv
    return f, g


def test_transport_products_against_plan_sums_and_gradient():
    x, y, a, b, _ = small(23, 17, 3, 11)
    eps = float(dense_cost(x, y).max()) / 8.0
    f, g = oracle.potentials(x, y, a, b, eps, 5)
    # P 1 and P^T 1 against the C oracle's plan sums (an independent code path)
    np.testing.assert_allclose(oracle.transport_apply(x, y, a, b, eps, f, g, np.ones(17)),
                               oracle.plan_row_sums(x, y, a, b, eps, f, g), rtol=1e-12)
    np.testing.assert_allclose(oracle.transport_apply_t(x, y, a, b, eps, f, g, np.ones(23)),
                               oracle.plan_col_sums(x, y, a, b, eps, f, g), rtol=1e-12)
    # P Y at the plan of (F(g), g) gives the gradient 2 (a x - P Y)
    ft = oracle.lse_update(x, y, b, g, eps)
    PY = oracle.transport_apply(x, y, a, b, eps, ft, g, y)
    np.testing.assert_allclose(2.0 * (a[:, None] * x - PY), oracle.grad_x(x, y, a, b, eps, g),
                               rtol=1e-10, atol=1e-13)


@pytest.mark.parametrize("n,m,d,seed,div", [(12, 10, 2, 12, 4.0), (9, 14, 3, 13, 2.0)])
def test_hvp_matches_gradient_finite_differences(n, m, d, seed, div):
    """The derivative of the converged gradient along v, by central differences of two
    fully converged solves at x +- h v."""
    x, y, a, b, _ = small(n, m, d, seed)
    eps = float(dense_cost(x, y).max()) / div
    v = np.random.default_rng(seed).standard_normal(x.shape)
    h = 1e-4

    def grad_at(xx):
        _, g = converged(xx, y, a, b, eps)
        return oracle.grad_x(xx, y, a, b, eps, g)

    fd = (grad_at(x + h * v) - grad_at(x - h * v)) / (2.0 * h)
    _, g = converged(x, y, a, b, eps)
    hv = oracle.hvp(x, y, a, b, eps, g, v)
    np.testing.assert_allclose(hv, fd, rtol=1e-5, atol=1e-6 * np.abs(fd).max())


def test_hvp_is_symmetric_and_gauge_invariant():
    x, y, a, b, _ = small(15, 11, 2, 14)
    eps = float(dense_cost(x, y).max()) / 5.0
    _, g = converged(x, y, a, b, eps)
    rng = np.random.default_rng(3)
    u, v = rng.standard_normal(x.shape), rng.standard_normal(x.shape)
    Hu = oracle.hvp(x, y, a, b, eps, g, u)
    Hv = oracle.hvp(x, y, a, b, eps, g, v)
    assert (u * Hv).sum() == pytest.approx((v * Hu).sum(), rel=1e-9, abs=1e-14)
    # F(g + c) = F(g) - c: the plan, hence H v, does not move
    np.testing.assert_allclose(oracle.hvp(x, y, a, b, eps, g + 0.37, v), Hv, rtol=1e-9,
                               atol=1e-12 * np.abs(Hv).max())


def test_hvp_large_eps_limit():
    """As eps grows the plan tends to a (x) b, which does not depend on x, and
    H v -> 2 a v, with an O(1/eps) remainder."""
    x, y, a, b, _ = small(10, 12, 2, 15)
    v = np.random.default_rng(4).standard_normal(x.shape)
    errs = []
    for eps in (1e2, 1e3, 1e4):
        _, g = converged(x, y, a, b, eps)
        errs.append(np.abs(oracle.hvp(x, y, a, b, eps, g, v) - 2.0 * a[:, None] * v).max())
    assert errs[2] < errs[1] < errs[0]
    assert errs[2] < 1e-3 * np.abs(2.0 * a[:, None] * v).max()
    assert errs[1] / errs[2] == pytest.approx(10.0, rel=0.2)


# --- the cosine cost -------------------------------------------------------------------------

def cosine_cost_matrix(x, y):
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    return 1.0 - (x @ y.T) / np.outer(np.linalg.norm(x, axis=1), np.linalg.norm(y, axis=1))


def test_cosine_matches_scaling_on_the_cosine_matrix():
    """Sinkhorn-Knopp on exp(-(1 - cos)/eps), computed from the cosines directly."""
    x, y, a, b, _ = small(19, 23, 4, 21)
    C = cosine_cost_matrix(x, y)
    eps = 0.05
    K = np.exp(-C / eps)
    v = b.copy()
    for _ in range(7):
        Kv = K @ v
        u = a / Kv
        Ktu = K.T @ u
        v = b / Ktu
    xs, ys = oracle.cosine_inputs(x, y)
    f, g = oracle.potentials(xs, ys, a, b, eps, 7)
    np.testing.assert_allclose(f, -eps * np.log(Kv), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(g, -eps * np.log(Ktu), rtol=1e-11, atol=1e-13)
    # the identity behind it
    np.testing.assert_allclose(dense_cost(xs, ys), C, rtol=1e-12, atol=1e-14)


def test_cosine_gradient_matches_finite_differences():
    x, y, a, b, _ = small(11, 9, 3, 22)
    eps = 0.1
    # a direction not drawn like x (the same draws would be parallel to each point, along
    # which the cosine cost does not move)
    v = np.random.default_rng(1022).standard_normal(x.shape)
    h = 1e-5

    def loss_at(xx):
        xs, ys = oracle.cosine_inputs(xx, y)
        f, g = converged(xs, ys, a, b, eps)
        return oracle.cost(xs, ys, a, b, eps, f, g)

    fd = (loss_at(x + h * v) - loss_at(x - h * v)) / (2.0 * h)
    xs, ys = oracle.cosine_inputs(x, y)
    _, g = converged(xs, ys, a, b, eps)
    gr = oracle.grad_x_cosine(x, y, a, b, eps, g)
    assert (gr * v).sum() == pytest.approx(fd, rel=1e-6, abs=1e-12)
    # the gradient is orthogonal to each point: scaling a point leaves its cosines alone
    np.testing.assert_allclose((gr * x).sum(axis=1), 0.0, atol=1e-12)


# --- the debiased divergence ---------------------------------------------------------------

CONV = dict(stop_mode="marginal", stop_tol=1e-13, stop_check_every=10, stop_max_iter=20000)


@pytest.mark.parametrize("seed", [30, 31, 32])
def test_divergence_is_nonnegative_and_zero_on_equal_clouds(seed):
    """At convergence the Sinkhorn divergence of the squared-Euclidean cost (a positive
    Gibbs kernel) is nonnegative, and zero for equal measures (Feydy et al. 2019, cited
    among the FS2 page's references for the debiased loss)."""
    x, y, a, b, _ = small(13, 17, 2, seed)
    eps = float(dense_cost(x, y).max()) / 6.0
    assert oracle.divergence(x, y, a, b, eps, **CONV) > 0.0
    assert abs(oracle.divergence(x, x, a, a, eps, **CONV)) < 1e-12


def test_divergence_large_eps_limit():
    """As eps grows each plan tends to the product of the marginals, and
    S -> int C d(a b) - int C d(a a)/2 - int C d(b b)/2 = |mean_a x - mean_b y|^2."""
    x, y, a, b, _ = small(10, 12, 3, 33)
    mx = (a[:, None] * x).sum(0) / a.sum()
    my = (b[:, None] * y).sum(0) / b.sum()
    target = float(((mx - my) ** 2).sum())
    errs = [abs(oracle.divergence(x, y, a, b, eps, **CONV) - target) for eps in (1e2, 1e3)]
    assert errs[1] < errs[0] and errs[1] < 1e-2 * target


def test_divergence_gradients_match_finite_differences():
    x, y, a, b, _ = small(9, 8, 2, 34)
    eps = float(dense_cost(x, y).max()) / 4.0
    rng = np.random.default_rng(340)
    vx, vy = rng.standard_normal(x.shape), rng.standard_normal(y.shape)
    h = 1e-5
    _, gx, gy = oracle.divergence(x, y, a, b, eps, grads=True, **CONV)
    fdx = (oracle.divergence(x + h * vx, y, a, b, eps, **CONV)
           - oracle.divergence(x - h * vx, y, a, b, eps, **CONV)) / (2 * h)
    fdy = (oracle.divergence(x, y + h * vy, a, b, eps, **CONV)
           - oracle.divergence(x, y - h * vy, a, b, eps, **CONV)) / (2 * h)
    assert (gx * vx).sum() == pytest.approx(fdx, rel=1e-6, abs=1e-11)
    assert (gy * vy).sum() == pytest.approx(fdy, rel=1e-6, abs=1e-11)
