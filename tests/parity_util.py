"""Shared helpers of the GPU parity tests: moving seeded inputs to the device and the
tolerances the comparisons use.

Tolerances (float32 streaming path against the float64 oracle):
  potentials  |f - f_ref| <= 1e-4 * max(1, |f_ref|) elementwise;
  cost        |D - D_ref| <= 1e-4 * max(1, |D_ref|);
  gradient    max_i |grad_i - grad_ref_i| <= 1e-4 * max|grad_ref| (a max-norm bound: every
              entry against the largest entry) on the float32 path, whose measured worst
              case on the three smaller configurations is 6.2e-6; per row also
              |grad_i - grad_ref_i| <= 1e-3 * 2 a_i sqrt(eps) where a test asks for it (the
              row's natural scale: 2 a_i times the width of the entropic kernel; measured
              worst 4.4e-5). The tensor-core path (d > 16) stores the plan weights as fp16,
              each off by at most 2^-11 relative, which moves the barycentre T_i by at most
              2^-11 of the row's mean |y_j - T_i|: 1e-3 of max|grad_ref| on small problems
              and 5e-3 (the tensor-core bar) on the 50k-point configuration.
The residual norms are computed from plan marginals r_i = a_i 2^E_i whose exponent E_i
carries the float32 rounding of the biased scores s_ij (|s| <= kappa * S with S the largest
squared norm of the centred points, kappa = log2(e)/eps). A few roundings of relative size
2^-24 each give |dE| <= ~8 * 2^-24 * kappa * S, so |r_i - r_ref_i| <= r_i * ln2 * |dE|, and the
residual norms agree to that bound times the mass (plus 1e-3 relative).
"""
import math

import numpy as np

try:
    import torch
except ImportError:  # pragma: no cover
    torch = None


def dev(arr):
    return torch.from_numpy(np.ascontiguousarray(arr)).cuda()


def inputs(w):
    return dev(w.x), dev(w.y), dev(w.a), dev(w.b)


def assert_potential_close(got, ref, name="f", rel=1e-4):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    tol = rel * np.maximum(1.0, np.abs(ref))
    err = np.abs(got - ref)
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, (f"{name}: {bad.size}/{ref.size} outside tolerance; worst index "
                           f"{int(np.argmax(err / tol))}: got {got[np.argmax(err / tol)]!r} "
                           f"ref {ref[np.argmax(err / tol)]!r} (max err {err.max():.3e})")


def assert_cost_close(got, ref, rel=1e-4):
    assert abs(got - ref) <= rel * max(1.0, abs(ref)), f"cost {got!r} vs oracle {ref!r}"


GRAD_REL = 1e-4     # float32 path
GRAD_REL_TC = 1e-3  # tensor-core path (d > 16), small problems


def grad_rel(d: int) -> float:
    return GRAD_REL if d <= 16 else GRAD_REL_TC


def assert_grad_close(got, ref, rel=GRAD_REL, row_scale=None, row_rel=1e-3):
    """max|got - ref| <= rel max|ref|; with row_scale (one value per row), also
    |got_i - ref_i| <= row_rel row_scale_i for every row i."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = max(np.abs(ref).max(), 1e-30)
    err = np.abs(got - ref).max()
    assert err <= rel * scale, f"grad max err {err:.3e} vs {rel:.0e} * {scale:.3e}"
    if row_scale is not None:
        e = np.abs(got - ref).reshape(len(ref), -1).max(1) / np.asarray(row_scale, np.float64)
        assert e.max() <= row_rel, f"grad row {int(np.argmax(e))}: err / row scale {e.max():.3e}"


def grad_row_scale(w, rows=None):
    """2 a_i sqrt(eps) per row (all rows, or the given ones)."""
    a = np.asarray(w.a, np.float64)
    if rows is not None:
        a = a[np.asarray(rows)]
    return 2.0 * a * math.sqrt(w.eps)


def score_scale(w) -> float:
    """kappa * S: the largest |s| magnitude of the float32 scores (centred clouds)."""
    x = w.x.astype(np.float64)
    y = w.y.astype(np.float64)
    c = (x.sum(0) + y.sum(0)) / (x.shape[0] + y.shape[0])
    s = max(((x - c) ** 2).sum(1).max(), ((y - c) ** 2).sum(1).max())
    return math.log2(math.e) / w.eps * 4.0 * max(s, 1e-30)


def residual_tolerance(w) -> float:
    """Absolute tolerance of the residual norms (see the module docstring)."""
    mass = float(np.asarray(w.a, np.float64).sum())
    return 8.0 * 2.0 ** -24 * score_scale(w) * math.log(2.0) * mass * 4.0 + 1e-7 * mass
