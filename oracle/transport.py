"""fp64 dense transport products and the Hessian-vector product -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
use this module; it shares no code with the CUDA library. Everything here forms the
explicit N x M plan in numpy and is meant for problems where that fits in memory.

What it computes (FlashSinkhorn summary, section 3, "Differentiation and Second-Order
Optimization": transport-matrix application, and a Hessian-vector product decomposed into
transport-vector and transport-matrix products; the pages give no formula for the HVP, so
the derivation below is ours, from the optimality conditions):

* ``plan(x, y, a, b, eps, f, g)``: P_ij = a_i b_j exp((f_i + g_j - C_ij)/eps),
  C_ij = |x_i - y_j|^2.
* ``transport_apply`` / ``transport_apply_t``: P U (U of shape (M, k)) and P^T W
  (W of shape (N, k)), the definition written out.
* ``hvp(x, y, a, b, eps, g, v)``: the derivative of the gradient
  G_i(x) = sum_j P_ij 2 (x_i - y_j) along v (one vector v_i per point x_i), P being the
  optimal plan, which moves with x through C and through the potentials. At the fixed
  point (sum_j P_ij = a_i, sum_i P_ij = b_j) differentiation gives, with
  dC_ij = 2 (x_i - y_j).v_i and dP_ij = P_ij (df_i + dg_j - dC_ij)/eps:
      a_i df_i + sum_j P_ij dg_j = r_i = sum_j P_ij dC_ij,
      sum_i P_ij df_i + b_j dg_j = s_j = sum_i P_ij dC_ij,
      (H v)_i = 2 a_i v_i + (2/eps) sum_j P_ij (x_i - y_j) (df_i + dg_j - dC_ij).
  P is the plan of (F(g), g), whose rows sum to a exactly (the plan the gradient uses);
  the system is written with the plan's own marginals, diag(P 1) and diag(P^T 1), which
  equal diag(a) and diag(b) at a converged g and make it positive semi-definite:
  (u, w) M (u, w) = sum_ij P_ij (u_i + w_j)^2. It is singular along (1, -1) (the gauge of
  the potentials), which the right-hand side respects (sum r = sum s); any solution gives
  the same H v, the exact Hessian-vector product at a converged g.
"""
from __future__ import annotations

import numpy as np


def _d(v):
    return np.asarray(v, dtype=np.float64)


def cost_matrix(x, y) -> np.ndarray:
    x, y = _d(x), _d(y)
    return ((x[:, None, :] - y[None, :, :]) ** 2).sum(-1)


def plan(x, y, a, b, eps: float, f, g) -> np.ndarray:
    C = cost_matrix(x, y)
    return _d(a)[:, None] * _d(b)[None, :] * np.exp((_d(f)[:, None] + _d(g)[None, :] - C) / eps)


def f_update(x, y, b, eps: float, g) -> np.ndarray:
    """F(g)_i = -eps log sum_j b_j exp((g_j - C_ij)/eps), with the maximum taken out."""
    C = cost_matrix(x, y)
    b = _d(b)
    z = (_d(g)[None, :] - C) / eps
    with np.errstate(divide="ignore"):
        z = z + np.log(b)[None, :]
    zmax = z.max(axis=1, keepdims=True)
    return -eps * (zmax[:, 0] + np.log(np.exp(z - zmax).sum(axis=1)))


def transport_apply(x, y, a, b, eps: float, f, g, U) -> np.ndarray:
    """P U for U of shape (M,) or (M, k)."""
    return plan(x, y, a, b, eps, f, g) @ _d(U)


def transport_apply_t(x, y, a, b, eps: float, f, g, W) -> np.ndarray:
    """P^T W for W of shape (N,) or (N, k)."""
    return plan(x, y, a, b, eps, f, g).T @ _d(W)


def hvp(x, y, a, b, eps: float, g, v) -> np.ndarray:
    """(H v)_i at the plan of (F(g), g); v has the shape of x."""
    x, y, a, b, v = _d(x), _d(y), _d(a), _d(b), _d(v)
    ft = f_update(x, y, b, eps, g)
    P = plan(x, y, a, b, eps, ft, g)
    diff = x[:, None, :] - y[None, :, :]                 # (N, M, d): x_i - y_j
    dC = 2.0 * np.einsum("ijk,ik->ij", diff, v)          # 2 (x_i - y_j).v_i
    r = (P * dC).sum(axis=1)
    s = (P * dC).sum(axis=0)
    n, m = P.shape
    M = np.zeros((n + m, n + m))
    M[:n, :n] = np.diag(P.sum(axis=1))
    M[:n, n:] = P
    M[n:, :n] = P.T
    M[n:, n:] = np.diag(P.sum(axis=0))
    sol = np.linalg.lstsq(M, np.concatenate([r, s]), rcond=None)[0]
    df, dg = sol[:n], sol[n:]
    w = P * (df[:, None] + dg[None, :] - dC)             # P_ij (df_i + dg_j - dC_ij)
    return 2.0 * a[:, None] * v + (2.0 / eps) * np.einsum("ij,ijk->ik", w, diff)
