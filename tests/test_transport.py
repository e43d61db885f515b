"""GPU parity of the transport products (fs_transport_apply) and the Hessian-vector product
(fs_hvp) against the fp64 oracle's dense definitions, and of the screened HVP against the
unscreened one on a clustered problem."""
import numpy as np
import pytest
import torch

import oracle
import streaming_sinkhorn_b200 as fs
from streaming_sinkhorn_b200 import workloads
from tests.parity_util import dev, inputs

pytestmark = pytest.mark.gpu


def problem(n, m, d, eps, seed):
    return workloads.random_small(n, m, d, seed=seed, eps=eps, n_iters=8)


def close(got, ref, rel):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = max(np.abs(ref).max(), 1e-30)
    err = np.abs(got - ref).max()
    assert err <= rel * scale, f"max err {err:.3e} vs {rel:.0e} * {scale:.3e}"


# Relative bar of a transport product against the oracle's dense one. The float32 path
# (d <= 16) meets 1e-4 of the largest entry. The tensor-core path (d > 16) forms
# P u / (P 1) with the plan weights rounded to fp16 (2^-11 relative each) and u to a
# [hi | lo] fp16 pair (2^-22 relative): each entry moves by at most 2^-11 of the row's
# mean |u_j - (P u)_i / (P 1)_i| (below max|u|) times the row mass, which bounds the error
# by 2^-11 max|u| a_i against entries of size ~ a_i |u|: 1e-3 of the largest entry.
TRANSPORT_REL = {False: 1e-4, True: 1e-3}


@pytest.mark.parametrize("k", [1, 3, 5, 16, 20])
@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("shape", [(300, 257, 2, 0.1), (129, 700, 3, 0.05), (200, 150, 8, 0.5),
                                   (90, 100, 16, 1.0), (200, 170, 32, 4.0), (130, 300, 64, 8.0),
                                   (150, 140, 256, 32.0)],
                         ids=lambda s: "n{}-m{}-d{}".format(*s[:3]))
def test_transport_apply_matches_dense_plan(shape, transpose, k):
    n, m, d, eps = shape
    w = problem(n, m, d, eps, seed=n + m + d + k)
    x, y, a, b = inputs(w)
    f, g = oracle.potentials(w.x, w.y, w.a, w.b, w.eps, 5)
    f32, g32 = f.astype(np.float32), g.astype(np.float32)
    rng = np.random.default_rng(k)
    u = rng.standard_normal(((n if transpose else m), k)).astype(np.float32)
    out = fs.transport_apply(x, y, dev(f32), dev(g32), dev(u), a, b, eps=w.eps,
                             transpose=transpose).cpu().numpy()
    fn = oracle.transport_apply_t if transpose else oracle.transport_apply
    ref = fn(w.x, w.y, w.a, w.b, w.eps, f32, g32, u)
    close(out, ref, TRANSPORT_REL[d > 16])


def test_transport_apply_vector_form():
    w = problem(100, 80, 3, 0.2, seed=5)
    x, y, a, b = inputs(w)
    f, g = oracle.potentials(w.x, w.y, w.a, w.b, w.eps, 5)
    f32, g32 = f.astype(np.float32), g.astype(np.float32)
    u = np.random.default_rng(1).standard_normal(80).astype(np.float32)
    out = fs.transport_apply(x, y, dev(f32), dev(g32), dev(u), a, b, eps=w.eps)
    assert out.shape == (100,)
    close(out.cpu().numpy(), oracle.transport_apply(w.x, w.y, w.a, w.b, w.eps, f32, g32, u), 1e-4)


# Bar of the HVP against the oracle, relative to the largest entry and, as a whole vector,
# in the 2-norm. fp32 conjugate gradients return an iterate at a relative residual of a few
# 1e-7 (the fp32 floor; reported by fs_hvp) and the transport passes are accurate to fp32
# rounding, so the entries agree to ~1e-5 of the largest (measured worst 1.1e-5); 1e-4
# leaves ten times that.
HVP_TOL = 1e-4
# d > 16: every transport product of the solve and the difference pass carry the fp16
# rounding of the plan weights (2^-11 relative each, see TRANSPORT_REL); the tensor-core bar.
HVP_TOL_TC = 5e-3


@pytest.mark.parametrize("shape", [(120, 90, 2, 0.3), (250, 300, 3, 0.1), (80, 70, 8, 1.0),
                                   (120, 100, 32, 4.0), (90, 110, 64, 8.0)],
                         ids=lambda s: "n{}-m{}-d{}".format(*s[:3]))
def test_hvp_matches_oracle(shape):
    n, m, d, eps = shape
    w = problem(n, m, d, eps, seed=7 * n + m)
    x, y, a, b = inputs(w)
    # the HVP is defined at any g (the plan of (F(g), g)); both sides use the same one,
    # near enough to convergence that the system is well conditioned (fp32 CG)
    _, g = oracle.potentials(w.x, w.y, w.a, w.b, w.eps, 400)
    g32 = g.astype(np.float32)
    v = np.random.default_rng(n).standard_normal((n, d)).astype(np.float32)
    hv, rep = fs.hvp(x, y, dev(g32), dev(v), a, b, eps=w.eps, cg_max_iter=500, cg_tol=1e-7)
    ref = oracle.hvp(w.x, w.y, w.a, w.b, w.eps, g32, v)
    assert rep["cg_iters"] >= 1
    hv = hv.cpu().numpy().astype(np.float64)
    tol = HVP_TOL if d <= 16 else HVP_TOL_TC
    close(hv, ref, tol)
    assert np.linalg.norm(hv - ref) <= tol * np.linalg.norm(ref)




def test_hvp_is_symmetric_on_the_gpu():
    """u.(Hv) = v.(Hu) (the Hessian is symmetric) and both equal the oracle's value.

    Error model: the GPU's Hv is within HVP_TOL |H_ref v|_2 of the oracle's in the 2-norm (the
    bar of test_hvp_matches_oracle), so by Cauchy-Schwarz |u.(Hv) - u.(H_ref v)| <= HVP_TOL
    |u|_2 |H_ref v|_2, and the GPU's asymmetry |u.(Hv) - v.(Hu)| is at most that bound for
    (u, v) plus the one for (v, u) plus the oracle's own (fp64) asymmetry. u is taken
    correlated with v (u = v + w / 2), so that u.(Hv) ~ v.(Hv) > 0 (H is positive
    semi-definite) and the bound is well under 1e-2 of the value, while a dropped or
    one-sided term of H changes it by O(1).
    """
    w = problem(200, 180, 3, 0.2, seed=17)
    x, y, a, b = inputs(w)
    _, g = oracle.potentials(w.x, w.y, w.a, w.b, w.eps, 400)
    g32 = g.astype(np.float32)
    gd = dev(g32)
    rng = np.random.default_rng(2)
    v = rng.standard_normal((200, 3)).astype(np.float32)
    u = (v + 0.5 * rng.standard_normal((200, 3))).astype(np.float32)
    hu, _ = fs.hvp(x, y, gd, dev(u), a, b, eps=w.eps, cg_max_iter=500, cg_tol=1e-7)
    hv, _ = fs.hvp(x, y, gd, dev(v), a, b, eps=w.eps, cg_max_iter=500, cg_tol=1e-7)
    hu, hv = hu.cpu().numpy().astype(np.float64), hv.cpu().numpy().astype(np.float64)
    hu_ref = oracle.hvp(w.x, w.y, w.a, w.b, w.eps, g32, u)
    hv_ref = oracle.hvp(w.x, w.y, w.a, w.b, w.eps, g32, v)
    u64, v64 = u.astype(np.float64), v.astype(np.float64)
    b_uv = HVP_TOL * np.linalg.norm(u64) * np.linalg.norm(hv_ref)
    b_vu = HVP_TOL * np.linalg.norm(v64) * np.linalg.norm(hu_ref)
    ref_uv, ref_vu = float((u64 * hv_ref).sum()), float((v64 * hu_ref).sum())
    lhs, rhs = float((u64 * hv).sum()), float((v64 * hu).sum())
    assert abs(ref_uv - ref_vu) <= 1e-9 * abs(ref_uv)  # the oracle is symmetric
    assert b_uv + b_vu <= 1e-2 * abs(ref_uv)  # the check can see an O(1) asymmetry
    assert abs(lhs - ref_uv) <= b_uv, (lhs, ref_uv, b_uv)
    assert abs(rhs - ref_vu) <= b_vu, (rhs, ref_vu, b_vu)
    assert abs(lhs - rhs) <= b_uv + b_vu + abs(ref_uv - ref_vu), (lhs, rhs)


def test_hvp_screened_equals_dense():
    """Screened and unscreened transport passes differ by fp32 rounding (at eps = 2e-4 the
    fp32 potentials alone fix each plan entry to ~1e-4); conjugate gradients stopped early
    amplify that, so both solves run until they stagnate at the same residual level."""
    w = workloads.clustered_cube(n=16384, seed=31, n_iters=10, eps=2e-4)
    x, y, a, b = inputs(w)
    f, g = fs.potentials(x, y, a, b, eps=w.eps, n_iters=10)
    v = torch.from_numpy(np.random.default_rng(3).standard_normal((w.n, 3)).astype(np.float32)).cuda()
    out = {}
    for screening in (False, True):
        fs.screening_enable(screening)
        try:
            hv, rep = fs.hvp(x, y, g, v, a, b, eps=w.eps, cg_max_iter=1000, cg_tol=1e-5)
        finally:
            fs.screening_enable(True)
        out[screening] = (hv.cpu().numpy(), rep)
    assert out[True][1]["cg_rel_residual"] < 2e-3 and out[False][1]["cg_rel_residual"] < 2e-3
    close(out[True][0], out[False][0], 5e-3)


@pytest.mark.parametrize("k", [3, 16])
@pytest.mark.parametrize("transpose", [False, True])
def test_transport_apply_screened_equals_dense(k, transpose):
    """On a clustered problem the screened products (tile screening and the 16-point group
    skip, 4- and 16-channel payload passes) agree with the unscreened ones: every term left
    out is below 2^-(24 + log2 M) of its row's largest plan entry."""
    w = workloads.clustered_cube(n=16384, seed=32, n_iters=6)
    x, y, a, b = inputs(w)
    f, g = fs.potentials(x, y, a, b, eps=w.eps, n_iters=6)
    u = torch.from_numpy(np.random.default_rng(k).standard_normal((w.n, k)).astype(np.float32)).cuda()
    out = {}
    for screening in (False, True):
        fs.screening_enable(screening)
        try:
            out[screening] = fs.transport_apply(x, y, f, g, u, a, b, eps=w.eps,
                                                transpose=transpose).cpu().numpy()
        finally:
            fs.screening_enable(True)
    close(out[True], out[False], 1e-4)
