"""fp64 CPU oracle for streaming log-domain Sinkhorn -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package. The product path (the CUDA library and its Python binding)
never imports, links or calls it, and it shares no code with that path.

The arithmetic lives in ``oracle.c`` (plain C + OpenMP, float64). This module only
marshals numpy arrays into it, plus the residual norms, which are a plain numpy
reduction of the plan marginals that ``oracle.c`` returns.

Each function names the passage of the pages it follows:

* ``lse_update``  -- one f- or g-update, FlashSinkhorn summary, Methodology section 1.
* ``potentials``  -- the alternating fixed-count schedule, SinkSLOT README API
  Reference (variant="alternating", stop_mode="fixed").
* ``cost``        -- the dual objective at (f, g), plan mass summed term by term.
* ``grad_x``      -- envelope gradient 2(a_i x_i - sum_j P_ij y_j), FlashSinkhorn summary
  section 3 and SinkSLOT README "Basic Usage".
* ``plan_row_sums`` / ``plan_col_sums`` / ``marginal_residual`` -- plan marginals and their
  deviation from (a, b), SinkSLOT README stop_mode "marginal".
* ``solve`` -- the general solve: symmetric (Jacobi) schedule and the marginal / potential
  stop modes, SinkSLOT README API Reference.
* ``cosine_inputs`` / ``grad_x_cosine`` -- the cosine cost C = 1 - cos(x, y), which equals
  |x/|x| - y/|y||^2 / 2: every function above applies to the normalised points scaled by
  sqrt(1/2), and the gradient with respect to x is the one with respect to those points
  times the normalisation's Jacobian (FlashSinkhorn summary: "cosine distance after
  normalization" shares the squared-Euclidean structure).
* ``divergence`` -- the debiased (Sinkhorn) divergence
  S = OT(a, b) - OT(a, a)/2 - OT(b, b)/2, each term the dual objective of its own solve with
  the same schedule, and its gradients: grad_x S = grad_x OT(x, y) - (G1 + G2)/2 with G1, G2
  the envelope gradients of OT(x, x) from each side (FlashSinkhorn 2 abstract and SinkSLOT
  README: the debiased "divergence" the losses report).
* ``transport_apply`` / ``transport_apply_t`` / ``hvp`` (numpy, ``transport.py``) -- the
  transport-vector and transport-matrix products and the Hessian-vector product of the
  loss, FlashSinkhorn summary section 3.

Pins: every function here is checked against closed forms, brute force and
invariants in ``tests/test_oracle_pins.py``; none is left unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .transport import hvp, plan, transport_apply, transport_apply_t  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    dp = ctypes.POINTER(ctypes.c_double)
    lp = ctypes.POINTER(ctypes.c_int64)
    i64, i32, dbl = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
    lib.oracle_lse_update.argtypes = [dp, i64, dp, i64, i32, dp, dp, dbl, lp, i64, dp]
    lib.oracle_potentials.argtypes = [dp, i64, dp, i64, i32, dp, dp, dbl, i32, dp, dp, dp]
    lib.oracle_plan_row_sums.argtypes = [dp, i64, dp, i64, i32, dp, dp, dbl, dp, dp, lp, i64, dp]
    lib.oracle_cost.argtypes = [dp, i64, dp, i64, i32, dp, dp, dbl, dp, dp, dp]
    lib.oracle_grad_x.argtypes = [dp, i64, dp, i64, i32, dp, dp, dbl, dp, lp, i64, dp]
    lib.oracle_solve.argtypes = [dp, i64, dp, i64, i32, dp, dp, dbl, i32, dbl, i32, i32, i32,
                                 dbl, i32, dp, dp, dp, ctypes.POINTER(ctypes.c_int32),
                                 ctypes.POINTER(ctypes.c_int32), dp]
    lib.oracle_set_threads.argtypes = [ctypes.c_int]
    lib.oracle_threads.restype = ctypes.c_int
    for fn in (lib.oracle_lse_update, lib.oracle_potentials, lib.oracle_plan_row_sums,
               lib.oracle_cost, lib.oracle_grad_x):
        fn.restype = ctypes.c_int
    _lib = lib
    return lib


class OracleError(ValueError):
    """Invalid arguments (code -1), mass mismatch or zero mass (-2), allocation failure (-3)."""

    def __init__(self, code: int):
        super().__init__({-1: "invalid argument", -2: "mass mismatch or zero total mass",
                          -3: "allocation failure"}.get(code, f"error {code}"))
        self.code = code


def _d(v) -> np.ndarray:
    return np.ascontiguousarray(v, dtype=np.float64)


def _p(arr: np.ndarray):
    return arr.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _rows(rows, count):
    if rows is None:
        return None, count
    r = np.ascontiguousarray(rows, dtype=np.int64)
    return r, int(r.shape[0])


def _rp(r):
    return None if r is None else r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


def _check(rc: int):
    if rc != 0:
        raise OracleError(rc)


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def threads() -> int:
    return int(_load().oracle_threads())


def lse_update(P, Q, wq, pot_q, eps: float, rows=None) -> np.ndarray:
    """out_k = -eps * log sum_j wq_j exp((pot_q_j - |P_i - Q_j|^2)/eps), i = rows[k]."""
    P, Q, wq, pot_q = _d(P), _d(Q), _d(wq), _d(pot_q)
    r, cnt = _rows(rows, P.shape[0])
    out = np.empty(cnt, dtype=np.float64)
    _check(_load().oracle_lse_update(_p(P), P.shape[0], _p(Q), Q.shape[0], P.shape[1], _p(wq),
                                     _p(pot_q), float(eps), _rp(r), cnt, _p(out)))
    return out


def potentials(x, y, a, b, eps: float, n_iters: int, g_init=None):
    """(f, g) after ``n_iters`` alternating iterations from g = g_init (zeros if None)."""
    x, y, a, b = _d(x), _d(y), _d(a), _d(b)
    n, m, d = x.shape[0], y.shape[0], x.shape[1]
    f = np.empty(n, dtype=np.float64)
    g = np.empty(m, dtype=np.float64)
    gi = None if g_init is None else _d(g_init)
    _check(_load().oracle_potentials(_p(x), n, _p(y), m, d, _p(a), _p(b), float(eps),
                                     int(n_iters), None if gi is None else _p(gi), _p(f), _p(g)))
    return f, g


def plan_row_sums(x, y, a, b, eps: float, f, g, rows=None) -> np.ndarray:
    """r_k = sum_j P_ij for i = rows[k] (all rows when None)."""
    x, y, a, b, f, g = _d(x), _d(y), _d(a), _d(b), _d(f), _d(g)
    r, cnt = _rows(rows, x.shape[0])
    out = np.empty(cnt, dtype=np.float64)
    _check(_load().oracle_plan_row_sums(_p(x), x.shape[0], _p(y), y.shape[0], x.shape[1], _p(a),
                                        _p(b), float(eps), _p(f), _p(g), _rp(r), cnt, _p(out)))
    return out


def plan_col_sums(x, y, a, b, eps: float, f, g, cols=None) -> np.ndarray:
    """c_k = sum_i P_ij for j = cols[k]: the row sums of the transposed problem."""
    return plan_row_sums(y, x, b, a, eps, g, f, rows=cols)


def cost(x, y, a, b, eps: float, f, g) -> float:
    """Dual objective <f,a> + <g,b> - eps*(sum_ij P_ij - m_a m_b)."""
    x, y, a, b, f, g = _d(x), _d(y), _d(a), _d(b), _d(f), _d(g)
    out = np.zeros(1, dtype=np.float64)
    _check(_load().oracle_cost(_p(x), x.shape[0], _p(y), y.shape[0], x.shape[1], _p(a), _p(b),
                               float(eps), _p(f), _p(g), _p(out)))
    return float(out[0])


def grad_x(x, y, a, b, eps: float, g, rows=None) -> np.ndarray:
    """Envelope gradient rows: 2(a_i x_i - sum_j Pt_ij y_j), Pt built from ft = F(g)."""
    x, y, a, b, g = _d(x), _d(y), _d(a), _d(b), _d(g)
    r, cnt = _rows(rows, x.shape[0])
    out = np.empty((cnt, x.shape[1]), dtype=np.float64)
    _check(_load().oracle_grad_x(_p(x), x.shape[0], _p(y), y.shape[0], x.shape[1], _p(a), _p(b),
                                 float(eps), _p(g), _rp(r), cnt, _p(out)))
    return out


def marginal_residual(x, y, a, b, eps: float, f, g) -> np.ndarray:
    """[L1(r - a), Linf(r - a), L1(c - b), Linf(c - b)] with r = P 1 and c = P^T 1."""
    r = plan_row_sums(x, y, a, b, eps, f, g)
    c = plan_col_sums(x, y, a, b, eps, f, g)
    dr = np.abs(r - _d(a))
    dc = np.abs(c - _d(b))
    return np.array([dr.sum(), dr.max(), dc.sum(), dc.max()], dtype=np.float64)


VARIANTS = {"alternating": 0, "symmetric": 1}
STOP_MODES = {"fixed": 0, "marginal": 1, "potential": 2}


def solve(x, y, a, b, eps: float, *, n_iters: int = 200, variant: str = "alternating",
          alpha: float = 0.5, stop_mode: str = "fixed", stop_max_iter: int = 20000,
          stop_tol: float = 1e-6, stop_check_every: int = 5, g_init=None):
    """The general solve: (f, g, iters_run, converged, final_viol).

    converged is None and final_viol NaN under stop_mode "fixed".
    """
    x, y, a, b = _d(x), _d(y), _d(a), _d(b)
    n, m, d = x.shape[0], y.shape[0], x.shape[1]
    f = np.empty(n, dtype=np.float64)
    g = np.empty(m, dtype=np.float64)
    gi = None if g_init is None else _d(g_init)
    it = ctypes.c_int32(0)
    conv = ctypes.c_int32(0)
    viol = np.zeros(1, dtype=np.float64)
    _check(_load().oracle_solve(_p(x), n, _p(y), m, d, _p(a), _p(b), float(eps),
                                VARIANTS[variant], float(alpha), STOP_MODES[stop_mode],
                                int(n_iters), int(stop_max_iter), float(stop_tol),
                                int(stop_check_every), None if gi is None else _p(gi), _p(f),
                                _p(g), ctypes.byref(it), ctypes.byref(conv), _p(viol)))
    converged = None if conv.value < 0 else bool(conv.value)
    return f, g, int(it.value), converged, float(viol[0])


def cosine_inputs(x, y):
    """The points on which the squared-Euclidean cost is 1 - cos(x, y): sqrt(1/2) x / |x|."""
    x, y = _d(x), _d(y)
    s = np.sqrt(0.5)
    return (s * x / np.linalg.norm(x, axis=1, keepdims=True),
            s * y / np.linalg.norm(y, axis=1, keepdims=True))


def grad_x_cosine(x, y, a, b, eps: float, g, rows=None) -> np.ndarray:
    """Envelope gradient of OT_eps with respect to x under the cosine cost: the gradient
    with respect to u = sqrt(1/2) x / |x| times du/dx = sqrt(1/2) (I - e e^T) / |x|,
    e = x / |x|."""
    x = _d(x)
    xs, ys = cosine_inputs(x, y)
    gu = grad_x(xs, ys, a, b, eps, g, rows=rows)
    xr = x if rows is None else x[np.asarray(rows)]
    nrm = np.linalg.norm(xr, axis=1, keepdims=True)
    e = xr / nrm
    return np.sqrt(0.5) / nrm * (gu - e * (e * gu).sum(axis=1, keepdims=True))


def divergence(x, y, a, b, eps: float, grads: bool = False, **solve_options):
    """S = OT(x, y) - OT(x, x)/2 - OT(y, y)/2, each solved by ``solve`` with the same
    options; with ``grads`` also (grad_x S, grad_y S)."""
    x, y, a, b = _d(x), _d(y), _d(a), _d(b)
    fxy, gxy, *_ = solve(x, y, a, b, eps, **solve_options)
    fxx, gxx, *_ = solve(x, x, a, a, eps, **solve_options)
    fyy, gyy, *_ = solve(y, y, b, b, eps, **solve_options)
    value = (cost(x, y, a, b, eps, fxy, gxy) - 0.5 * cost(x, x, a, a, eps, fxx, gxx)
             - 0.5 * cost(y, y, b, b, eps, fyy, gyy))
    if not grads:
        return value
    gx = grad_x(x, y, a, b, eps, gxy) - 0.5 * (grad_x(x, x, a, a, eps, gxx)
                                               + grad_x(x, x, a, a, eps, fxx))
    gy = grad_x(y, x, b, a, eps, fxy) - 0.5 * (grad_x(y, y, b, b, eps, gyy)
                                               + grad_x(y, y, b, b, eps, fyy))
    return value, gx, gy
