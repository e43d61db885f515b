"""Streaming log-domain Sinkhorn on B200 (sm_100a): Python binding of include/fs.h.

Every function here only marshals arguments into the C ABI of ``libfs.so``; every step of
the computation runs in the library's CUDA kernels. PyTorch supplies device memory and
the current stream. There is no CPU path: the functions raise when the library or a
CUDA device is missing.

Conventions (SinkSLOT README, "Tensor Contract" and dtype table): x (N, d), y (M, d),
optional nonnegative weights a (N,), b (M,) (uniform when omitted), all float32 CUDA
tensors on one device; float64 raises ValueError because the fused kernels are
float32-only; a/b are used as given and sum(a) must equal sum(b) (ValueError otherwise);
zero weights are legal; N != M is allowed. Potentials are returned in cost units (f, g).
"""
from __future__ import annotations

import ctypes

from . import _lib

__all__ = ["potentials", "cost", "grad_x", "marginal_residual", "solve_host", "workspace_bytes",
           "workspace_invalidate",
           "FsError", "timing_enable", "timing_reset", "timing_get", "launch_count",
           "screening_enable", "solve", "transport_apply", "hvp", "SamplesLoss",
           "sinkhorn_divergence", "solve_multiscale"]


class FsError(RuntimeError):
    """A failed library call; ``status`` holds the fs_status name."""

    def __init__(self, status: int, detail: str = ""):
        self.status = _lib.STATUS.get(status, str(status))
        msg = _lib.load().fs_status_string(status).decode()
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


class FsValueError(FsError, ValueError):
    """Invalid inputs: bad shapes, weights, eps, iteration count or workspace."""


_INPUT_ERRORS = {1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 13}


def _raise(status: int):
    if status == 0:
        return
    if status in _INPUT_ERRORS:
        raise FsValueError(status)
    detail = _lib.load().fs_last_cuda_error().decode() if status == 12 else ""
    raise FsError(status, detail)


def _torch():
    import torch
    return torch


def _check_tensor(t, name, shape=None, device=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype == torch.float64:
        raise ValueError(f"{name} is float64: the fused kernels are float32-only")
    if t.dtype != torch.float32:
        raise TypeError(f"{name} must be float32, got {t.dtype}")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.contiguous()


class _Problem:
    """Validated tensors plus the fs_problem struct that points at them."""

    def __init__(self, x, y, a, b, eps, cost="sqeuclidean"):
        torch = _torch()
        if not isinstance(x, torch.Tensor) or x.dim() != 2:
            raise ValueError("x must be a 2-D tensor (N, d)")
        if not isinstance(y, torch.Tensor) or y.dim() != 2:
            raise ValueError("y must be a 2-D tensor (M, d)")
        self.x = _check_tensor(x, "x")
        self.device = self.x.device
        n, d = self.x.shape
        self.y = _check_tensor(y, "y", device=self.device)
        if self.y.shape[1] != d:
            raise ValueError(f"x has d={d} but y has d={self.y.shape[1]}")
        m = self.y.shape[0]
        self.a = None if a is None else _check_tensor(a, "a", (n,), self.device)
        self.b = None if b is None else _check_tensor(b, "b", (m,), self.device)
        self.n, self.m, self.d = int(n), int(m), int(d)
        self.eps = float(eps)
        if cost not in _lib.COSTS:
            raise ValueError(f"unknown cost {cost!r}: {sorted(_lib.COSTS)}")
        self.cost = cost
        self.s = _lib.fs_problem(self.x.data_ptr(), self.y.data_ptr(),
                                 None if self.a is None else self.a.data_ptr(),
                                 None if self.b is None else self.b.data_ptr(),
                                 self.n, self.m, self.d, self.eps, _lib.COSTS[cost])

    @property
    def ref(self):
        return ctypes.byref(self.s)

    def stream(self):
        return _torch().cuda.current_stream(self.device).cuda_stream

    def workspace(self):
        nbytes = workspace_bytes(self.n, self.m, self.d, self.device, cost=self.cost)
        # torch's caching allocator returns 512-byte aligned blocks
        return _torch().empty(max(nbytes, 1), dtype=_torch().uint8, device=self.device)


def workspace_bytes(n: int, m: int, d: int, device=None, cost: str = "sqeuclidean") -> int:
    """fs_workspace_bytes for an (n, m, d) problem on ``device`` (the current one if None)."""
    torch = _torch()
    lib = _lib.load()
    p = _lib.fs_problem(None, None, None, None, int(n), int(m), int(d), 1.0, _lib.COSTS[cost])
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        return int(lib.fs_workspace_bytes(ctypes.byref(p)))


def potentials(x, y, a=None, b=None, *, eps: float, ground_cost: str = "sqeuclidean",
               n_iters: int, g_init=None, out=None,
               workspace=None):
    """(f, g) after ``n_iters`` alternating f/g updates starting from g = g_init (or 0).

    FlashSinkhorn summary, Methodology section 1 (update), SinkSLOT README API Reference
    (alternating variant, fixed iteration count). ``out`` may pass preallocated (f, g).
    """
    torch = _torch()
    P = _Problem(x, y, a, b, eps, ground_cost)
    if out is None:
        f = torch.empty(P.n, dtype=torch.float32, device=P.device)
        g = torch.empty(P.m, dtype=torch.float32, device=P.device)
    else:
        f = _check_tensor(out[0], "f", (P.n,), P.device)
        g = _check_tensor(out[1], "g", (P.m,), P.device)
    gi = None if g_init is None else _check_tensor(g_init, "g_init", (P.m,), P.device)
    ws = P.workspace() if workspace is None else workspace
    _raise(_lib.load().fs_potentials(P.ref, int(n_iters), None if gi is None else gi.data_ptr(),
                                     f.data_ptr(), g.data_ptr(), ws.data_ptr(), ws.numel(),
                                     P.stream()))
    return f, g


def solve(x, y, a=None, b=None, *, eps: float, ground_cost: str = "sqeuclidean",
          n_iters: int = 200, variant: str = "alternating",
          alpha: float = 0.5, stop_mode: str = "fixed", stop_max_iter: int = 20000,
          stop_tol: float = 1e-6, stop_check_every: int = 5, g_init=None, out=None,
          workspace=None):
    """The general solve (fs_solve): (f, g, report).

    SinkSLOT README, API Reference: ``variant`` "alternating" (Gauss-Seidel) or "symmetric"
    (Jacobi, blended with ``alpha``); ``stop_mode`` "fixed" (``n_iters`` iterations),
    "marginal" or "potential" (at most ``stop_max_iter``, checked every
    ``stop_check_every`` against ``stop_tol``). ``report`` holds iters_run, converged (None
    under "fixed") and final_viol (NaN under "fixed").
    """
    torch = _torch()
    P = _Problem(x, y, a, b, eps, ground_cost)
    if out is None:
        f = torch.empty(P.n, dtype=torch.float32, device=P.device)
        g = torch.empty(P.m, dtype=torch.float32, device=P.device)
    else:
        f = _check_tensor(out[0], "f", (P.n,), P.device)
        g = _check_tensor(out[1], "g", (P.m,), P.device)
    gi = None if g_init is None else _check_tensor(g_init, "g_init", (P.m,), P.device)
    if variant not in _lib.VARIANTS or stop_mode not in _lib.STOP_MODES:
        raise ValueError(f"unknown variant {variant!r} or stop_mode {stop_mode!r}")
    opt = _lib.fs_solve_options(int(n_iters), _lib.VARIANTS[variant], float(alpha),
                                _lib.STOP_MODES[stop_mode], int(stop_max_iter),
                                int(stop_check_every), float(stop_tol),
                                None if gi is None else gi.data_ptr())
    rep = _lib.fs_solve_report()
    ws = P.workspace() if workspace is None else workspace
    _raise(_lib.load().fs_solve(P.ref, ctypes.byref(opt), f.data_ptr(), g.data_ptr(),
                                ctypes.byref(rep), ws.data_ptr(), ws.numel(), P.stream()))
    report = {"iters_run": int(rep.iters_run),
              "converged": None if rep.converged < 0 else bool(rep.converged),
              "final_viol": float(rep.final_viol)}
    return f, g, report


def solve_multiscale(x, y, a=None, b=None, *, eps: float, cell_points: int = 8,
                     coarse_iters: int = 50,
                     max_rounds: int = 8, lift_tol: float = 0.0, lift_shrink: float = 0.5,
                     n_iters: int = 200, stop_mode: str = "fixed", stop_max_iter: int = 20000,
                     stop_tol: float = 1e-6, stop_check_every: int = 5, variant: str = "alternating",
                     alpha: float = 0.5, workspace=None):
    """Coarse-to-fine solve (fs_solve_multiscale): rounds on Morton cells of ``cell_points``
    consecutive points, lifts to
    the fine y checked by one fine iteration, then fs_solve from the accepted lift.
    Returns (f, g, report)."""
    torch = _torch()
    P = _Problem(x, y, a, b, eps)
    f = torch.empty(P.n, dtype=torch.float32, device=P.device)
    g = torch.empty(P.m, dtype=torch.float32, device=P.device)
    opt = _lib.fs_solve_options(int(n_iters), _lib.VARIANTS[variant], float(alpha),
                                _lib.STOP_MODES[stop_mode], int(stop_max_iter),
                                int(stop_check_every), float(stop_tol), None)
    mo = _lib.fs_multiscale_options(int(cell_points), int(coarse_iters), int(max_rounds),
                                    float(lift_tol), float(lift_shrink))
    rep = _lib.fs_multiscale_report()
    if workspace is None:
        nbytes = int(_lib.load().fs_multiscale_workspace_bytes(P.ref, int(cell_points)))
        if nbytes == 0:
            raise ValueError("the coarse-to-fine solve needs 1 <= d <= 16")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=P.device)
    _raise(_lib.load().fs_solve_multiscale(P.ref, ctypes.byref(opt), ctypes.byref(mo),
                                           f.data_ptr(), g.data_ptr(), ctypes.byref(rep),
                                           workspace.data_ptr(), workspace.numel(), P.stream()))
    fine = rep.fine
    report = {"rounds": int(rep.rounds), "coarse_iters": int(rep.coarse_iters),
              "lift_viol": float(rep.lift_viol),
              "fine": {"iters_run": int(fine.iters_run),
                       "converged": None if fine.converged < 0 else bool(fine.converged),
                       "final_viol": float(fine.final_viol)}}
    return f, g, report


def sinkhorn_divergence(x, y, a=None, b=None, *, eps: float, ground_cost: str = "sqeuclidean",
                        grads: bool = False, n_iters: int = 200, variant: str = "alternating",
                        alpha: float = 0.5, stop_mode: str = "fixed", stop_max_iter: int = 20000,
                        stop_tol: float = 1e-6, stop_check_every: int = 5, workspace=None):
    """Debiased divergence OT(a, b) - OT(a, a)/2 - OT(b, b)/2 (fs_divergence) as a 0-d
    float64 tensor; with ``grads`` also its gradients for x (N, d) and y (M, d)."""
    torch = _torch()
    P = _Problem(x, y, a, b, eps, ground_cost)
    opt = _lib.fs_solve_options(int(n_iters), _lib.VARIANTS[variant], float(alpha),
                                _lib.STOP_MODES[stop_mode], int(stop_max_iter),
                                int(stop_check_every), float(stop_tol), None)
    value = torch.empty((), dtype=torch.float64, device=P.device)
    gx = torch.empty((P.n, P.d), dtype=torch.float32, device=P.device) if grads else None
    gy = torch.empty((P.m, P.d), dtype=torch.float32, device=P.device) if grads else None
    if workspace is None:
        nbytes = int(_lib.load().fs_divergence_workspace_bytes(P.ref))
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=P.device)
    _raise(_lib.load().fs_divergence(P.ref, ctypes.byref(opt), value.data_ptr(),
                                     None if gx is None else gx.data_ptr(),
                                     None if gy is None else gy.data_ptr(), workspace.data_ptr(),
                                     workspace.numel(), P.stream()))
    return (value, gx, gy) if grads else value


def _transport_workspace(P):
    nbytes = int(_lib.load().fs_transport_workspace_bytes(P.ref))
    if nbytes == 0:
        raise ValueError("transport products need 1 <= d <= 16")
    return _torch().empty(nbytes, dtype=_torch().uint8, device=P.device)


def transport_apply(x, y, f, g, u, a=None, b=None, *, eps: float, ground_cost: str = "sqeuclidean",
                    transpose: bool = False,
                    workspace=None):
    """P u (u: (M,) or (M, k)) or, with ``transpose``, P^T u (u: (N,) or (N, k)), with
    P_ij = a_i b_j exp((f_i + g_j - |x_i - y_j|^2)/eps) streamed, never stored
    (fs_transport_apply; FlashSinkhorn summary section 3, transport-matrix application)."""
    torch = _torch()
    P = _Problem(x, y, a, b, eps, ground_cost)
    f = _check_tensor(f, "f", (P.n,), P.device)
    g = _check_tensor(g, "g", (P.m,), P.device)
    rows_in = P.n if transpose else P.m
    rows_out = P.m if transpose else P.n
    vec = u.dim() == 1
    u2 = u.reshape(-1, 1) if vec else u
    k = int(u2.shape[1])
    u2 = _check_tensor(u2, "u", (rows_in, k), P.device)
    out = torch.empty((rows_out, k), dtype=torch.float32, device=P.device)
    ws = _transport_workspace(P) if workspace is None else workspace
    _raise(_lib.load().fs_transport_apply(P.ref, f.data_ptr(), g.data_ptr(), 1 if transpose else 0,
                                          k, u2.data_ptr(), out.data_ptr(), ws.data_ptr(),
                                          ws.numel(), P.stream()))
    return out.reshape(-1) if vec else out


def hvp(x, y, g, v, a=None, b=None, *, eps: float, ground_cost: str = "sqeuclidean",
        cg_max_iter: int = 200, cg_tol: float = 1e-6,
        workspace=None):
    """Hessian-vector product of OT_eps with respect to x at the plan of (F(g), g), v of
    shape (N, d) (fs_hvp; FlashSinkhorn summary section 3). Returns (H v, report)."""
    torch = _torch()
    P = _Problem(x, y, a, b, eps, ground_cost)
    g = _check_tensor(g, "g", (P.m,), P.device)
    v = _check_tensor(v, "v", (P.n, P.d), P.device)
    out = torch.empty((P.n, P.d), dtype=torch.float32, device=P.device)
    opt = _lib.fs_hvp_options(int(cg_max_iter), float(cg_tol))
    rep = _lib.fs_hvp_report()
    ws = _transport_workspace(P) if workspace is None else workspace
    _raise(_lib.load().fs_hvp(P.ref, g.data_ptr(), v.data_ptr(), out.data_ptr(), ctypes.byref(opt),
                              ctypes.byref(rep), ws.data_ptr(), ws.numel(), P.stream()))
    return out, {"cg_iters": int(rep.cg_iters), "cg_rel_residual": float(rep.cg_rel_residual)}


def cost(x, y, f, g, a=None, b=None, *, eps: float, ground_cost: str = "sqeuclidean",
         workspace=None):
    """Dual objective <f,a> + <g,b> - eps (sum_ij P_ij - m_a m_b) as a 0-d float64 tensor."""
    torch = _torch()
    P = _Problem(x, y, a, b, eps, ground_cost)
    f = _check_tensor(f, "f", (P.n,), P.device)
    g = _check_tensor(g, "g", (P.m,), P.device)
    out = torch.empty((), dtype=torch.float64, device=P.device)
    ws = P.workspace() if workspace is None else workspace
    _raise(_lib.load().fs_cost(P.ref, f.data_ptr(), g.data_ptr(), out.data_ptr(), ws.data_ptr(),
                               ws.numel(), P.stream()))
    return out


def grad_x(x, y, g, a=None, b=None, *, eps: float, ground_cost: str = "sqeuclidean",
           out=None, workspace=None):
    """Envelope gradient 2 (a_i x_i - sum_j P_ij y_j) with the plan of (F(g), g), (N, d)."""
    torch = _torch()
    P = _Problem(x, y, a, b, eps, ground_cost)
    g = _check_tensor(g, "g", (P.m,), P.device)
    gr = (torch.empty((P.n, P.d), dtype=torch.float32, device=P.device) if out is None
          else _check_tensor(out, "out", (P.n, P.d), P.device))
    ws = P.workspace() if workspace is None else workspace
    _raise(_lib.load().fs_grad_x(P.ref, g.data_ptr(), gr.data_ptr(), ws.data_ptr(), ws.numel(),
                                 P.stream()))
    return gr


def marginal_residual(x, y, f, g, a=None, b=None, *, eps: float, ground_cost: str = "sqeuclidean",
                      marginals: bool = False,
                      workspace=None):
    """[sum|P1 - a|, max|P1 - a|, sum|P^T 1 - b|, max|P^T 1 - b|] (float64, device).

    With ``marginals=True`` also returns the plan marginals r = P 1 and c = P^T 1.
    """
    torch = _torch()
    P = _Problem(x, y, a, b, eps, ground_cost)
    f = _check_tensor(f, "f", (P.n,), P.device)
    g = _check_tensor(g, "g", (P.m,), P.device)
    out = torch.empty(4, dtype=torch.float64, device=P.device)
    r = torch.empty(P.n, dtype=torch.float32, device=P.device) if marginals else None
    c = torch.empty(P.m, dtype=torch.float32, device=P.device) if marginals else None
    ws = P.workspace() if workspace is None else workspace
    _raise(_lib.load().fs_marginal_residual(
        P.ref, f.data_ptr(), g.data_ptr(), out.data_ptr(), None if r is None else r.data_ptr(),
        None if c is None else c.data_ptr(), ws.data_ptr(), ws.numel(), P.stream()))
    return (out, r, c) if marginals else out


def solve_host(x, y, a=None, b=None, *, eps: float, n_iters: int, grad: bool = True,
               residual: bool = True, cost: bool = True, device=None, workspace=None, out=None,
               ground_cost: str = "sqeuclidean"):
    """One fs_solve_host call on host arrays (numpy or CPU tensors, float32).

    Copies the inputs to the device, solves, and copies f, g and the requested extras
    back. Pinned CPU tensors make the copies asynchronous. Returns a dict of CPU tensors.
    """
    torch = _torch()

    def host(t, name):
        if t is None:
            return None
        if not isinstance(t, torch.Tensor):
            t = torch.from_numpy(t)
        if t.dtype == torch.float64:
            raise ValueError(f"{name} is float64: the fused kernels are float32-only")
        if t.device.type != "cpu" or t.dtype != torch.float32:
            raise ValueError(f"{name} must be a float32 host array")
        return t.contiguous()

    xh, yh, ah, bh = host(x, "x"), host(y, "y"), host(a, "a"), host(b, "b")
    n, d = xh.shape
    m = yh.shape[0]
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    p = _lib.fs_problem(xh.data_ptr(), yh.data_ptr(), None if ah is None else ah.data_ptr(),
                        None if bh is None else bh.data_ptr(), n, m, d, float(eps),
                        _lib.COSTS[ground_cost])
    lib = _lib.load()
    with torch.cuda.device(dev):
        nbytes = int(lib.fs_solve_host_workspace_bytes(ctypes.byref(p)))
        ws = (torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev) if workspace is None
              else workspace)
        if out is None:
            pin = torch.cuda.is_available()
            out = {"f": torch.empty(n, dtype=torch.float32, pin_memory=pin),
                   "g": torch.empty(m, dtype=torch.float32, pin_memory=pin),
                   "grad_x": torch.empty((n, d), dtype=torch.float32, pin_memory=pin),
                   "cost": torch.empty(1, dtype=torch.float64, pin_memory=pin),
                   "residual": torch.empty(4, dtype=torch.float64, pin_memory=pin)}
        stream = torch.cuda.current_stream(dev).cuda_stream
        _raise(lib.fs_solve_host(ctypes.byref(p), int(n_iters), out["f"].data_ptr(),
                                 out["g"].data_ptr(), out["grad_x"].data_ptr() if grad else None,
                                 out["cost"].data_ptr() if cost else None,
                                 out["residual"].data_ptr() if residual else None, ws.data_ptr(),
                                 ws.numel(), stream))
    return out


def timing_enable(on: bool = True) -> None:
    _lib.load().fs_timing_enable(1 if on else 0)


def timing_reset() -> None:
    _lib.load().fs_timing_reset()


def screening_enable(on: bool = True) -> None:
    """Turns block screening on or off for later calls (fs_screening_enable)."""
    _lib.load().fs_screening_enable(1 if on else 0)


def workspace_invalidate(workspace) -> None:
    """Drops what ``workspace`` (a device uint8 tensor) remembers from earlier calls: the
    Morton order of the last clouds it sorted, which later calls on the same clouds reuse
    (fs_workspace_invalidate). Never needed for correct results."""
    torch = _torch()
    st = torch.cuda.current_stream(workspace.device).cuda_stream
    _raise(_lib.load().fs_workspace_invalidate(workspace.data_ptr(), workspace.numel(), st))


def launch_count() -> int:
    """Kernels launched by the library so far in this process (fs_launch_count)."""
    return int(_lib.load().fs_launch_count())


def timing_get() -> dict:
    t = _lib.fs_timing()
    _lib.load().fs_timing_get(ctypes.byref(t))
    return {name: {"launches": int(getattr(t, name).launches),
                   "total_ms": float(getattr(t, name).total_ms),
                   "pairs": float(getattr(t, name).pairs),
                   "evaluated": float(getattr(t, name).evaluated)}
            for name in ("lse_pass", "grad_pass", "marg_pass", "combine", "screen")}


from .loss import SamplesLoss  # noqa: E402  (uses the functions above)
