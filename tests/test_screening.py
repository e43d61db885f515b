"""Block screening on the GPU: a clustered problem solved with screening on and off gives
the same potentials, gradient and marginals to fp32 rounding, and the screened run
evaluates far fewer pairs. Screening drops only tiles whose terms are all below
2^-(24 + log2 M) of their rows' largest term, so any larger difference is a bug in the
bound, the kept-tile masks, the unit plan or the merge of a row block's units."""
import numpy as np
import pytest

import streaming_sinkhorn_b200 as fs
from streaming_sinkhorn_b200 import workloads
from tests.parity_util import assert_grad_close, assert_potential_close, dev, inputs

pytestmark = pytest.mark.gpu

# Gradient bar of screened against unscreened runs at small eps. The key biases kappa g
# reach ~1e3 log2 units there, so every weight 2^(z - m) carries the fp32 rounding of its
# exponent, ~8 * 2^-24 * 1e3 = 4.8e-4 log2 units, i.e. 3.3e-4 relative (times ln 2), which
# moves a row's barycentre by up to that fraction of the row's spread (of the order of
# |x_i - T_i| at small eps); two summation orders: 1e-3 of the largest entry. Screening's
# own omission (under 2^-24 of a row's mass) is far below it.
GRAD_REL_SMALL_EPS = 1e-3


def solve(w, screening):
    x, y, a, b = inputs(w)
    fs.screening_enable(screening)
    try:
        fs.timing_enable(True)
        fs.timing_reset()
        f, g = fs.potentials(x, y, a, b, eps=w.eps, n_iters=w.n_iters)
        t = fs.timing_get()
    finally:
        fs.timing_enable(False)
        fs.screening_enable(True)
    return f.cpu().numpy(), g.cpu().numpy(), t


def passes(w, f, g, screening):
    """The gradient, marginal and cost passes at given potentials."""
    x, y, a, b = inputs(w)
    fd, gd = dev(f), dev(g)
    fs.screening_enable(screening)
    try:
        gx = fs.grad_x(x, y, gd, a, b, eps=w.eps)
        res, r, c = fs.marginal_residual(x, y, fd, gd, a, b, eps=w.eps, marginals=True)
        cost = fs.cost(x, y, fd, gd, a, b, eps=w.eps).item()
    finally:
        fs.screening_enable(True)
    return gx.cpu().numpy(), r.cpu().numpy(), c.cpu().numpy(), res.cpu().numpy(), cost


@pytest.mark.parametrize("n,m", [(32768, 32768), (20000, 45000)])
def test_screened_equals_dense(n, m):
    # eps near the 2^20-point workload's, so that most key tiles are provably negligible
    w = workloads.clustered_cube(n=n, seed=11, n_iters=6, eps=1e-4)
    if m != n:  # unequal clouds: a second, independently seeded cloud for y
        import dataclasses
        w2 = workloads.clustered_cube(n=m, seed=12, n_iters=6, eps=w.eps)
        w = dataclasses.replace(w, y=w2.y, b=w2.b)
    fd, gd, td = solve(w, False)
    fsc, gsc, ts = solve(w, True)
    # Potentials in exponent units (kappa * f, the log2 of a weight). The biases kappa * g
    # reach ~1e3 here, so fp32 rounding (ulp ~1e-4) in two summation orders over six
    # iterations moves the worst row by ~2e-3; a wrongly dropped tile holding even 1 % of a
    # row's mass would move it by >= 1.4e-2, and one holding its main terms by O(1).
    kappa = 1.0 / (w.eps * np.log(2.0))
    df = np.abs(fsc.astype(np.float64) - fd).max() * kappa
    dg = np.abs(gsc.astype(np.float64) - gd).max() * kappa
    assert df < 1e-2 and dg < 1e-2, (df, dg)
    assert_potential_close(fsc, fd, "f", rel=1e-6)
    assert_potential_close(gsc, gd, "g", rel=1e-6)
    # the dense run evaluated every pair (padding included); the screened one far fewer
    lse_d, lse_s = td["lse_pass"], ts["lse_pass"]
    assert lse_d["evaluated"] >= lse_d["pairs"]
    assert lse_s["evaluated"] < 0.25 * lse_s["pairs"]
    assert ts["screen"]["launches"] > 0 and td["screen"]["launches"] == 0

    # the other passes, screened and dense, at the same potentials
    gxd, rd, cd, resd, costd = passes(w, fd, gd, False)
    gxs, rs, cs, ress, costs = passes(w, fd, gd, True)
    assert_grad_close(gxs, gxd, rel=GRAD_REL_SMALL_EPS)
    np.testing.assert_allclose(rs, rd, rtol=1e-3, atol=1e-7 * float(w.a.max()))
    np.testing.assert_allclose(cs, cd, rtol=1e-3, atol=1e-7 * float(w.b.max()))
    # the column residual sits at the rounding floor (g was just updated from these very
    # sums), where any change of summation order shows at ~1e-6 of the mass
    np.testing.assert_allclose(ress, resd, rtol=1e-3, atol=2e-5 * float(w.b.sum()))
    assert costs == pytest.approx(costd, rel=1e-4)


@pytest.mark.parametrize("d", [2, 5, 8])
def test_screened_equals_dense_other_dims(d):
    """Other widths: 16-bit Morton codes at d = 2, codes of the first three coordinates at
    d = 5 and 8 (so the anchors come from a projection of the points), ragged row blocks
    and key tiles (n, m not multiples of 64 and 256)."""
    w = workloads.mixture_pair(n=24001, m=30011, d=d, k=40, std=0.03, seed=13 + d, eps=1e-3,
                               n_iters=6, clip_unit_cube=True)
    fd, gd, td = solve(w, False)
    fsc, gsc, ts = solve(w, True)
    kappa = 1.0 / (w.eps * np.log(2.0))
    df = np.abs(fsc.astype(np.float64) - fd).max() * kappa
    dg = np.abs(gsc.astype(np.float64) - gd).max() * kappa
    assert df < 1e-2 and dg < 1e-2, (df, dg)
    assert ts["screen"]["launches"] > 0
    assert ts["lse_pass"]["evaluated"] < 0.9 * ts["lse_pass"]["pairs"]
    gxd, rd, cd, resd, costd = passes(w, fd, gd, False)
    gxs, rs, cs, ress, costs = passes(w, fd, gd, True)
    assert_grad_close(gxs, gxd, rel=GRAD_REL_SMALL_EPS)
    np.testing.assert_allclose(rs, rd, rtol=1e-3, atol=1e-7 * float(w.a.max()))
    assert costs == pytest.approx(costd, rel=1e-4)
