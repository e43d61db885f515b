"""A loss module in the style of the pages' ``SamplesLoss`` (SinkSLOT README, "Basic Usage"):
``loss(x, y)`` solves the entropic problem with the library's kernels and returns the dual
objective at the solution; its backward is the analytic envelope gradient of fs_grad_x,
with no differentiation through the iterations.

Only argument marshalling happens here: every number comes from the C ABI.
"""
from __future__ import annotations

from . import _torch, cost, grad_x, sinkhorn_divergence, solve


class _OTLoss:
    """Factory of the autograd function (built on first use, so importing the package
    does not import torch)."""

    fn = None
    div = None

    @classmethod
    def get(cls):
        if cls.fn is None:
            torch = _torch()

            class OTLossFunction(torch.autograd.Function):
                @staticmethod
                def forward(ctx, x, y, a, b, eps, ground_cost, options):
                    xd, yd = x.detach(), y.detach()
                    f, g, report = solve(xd, yd, a, b, eps=eps, ground_cost=ground_cost,
                                         **options)
                    value = cost(xd, yd, f, g, a, b, eps=eps, ground_cost=ground_cost)
                    ctx.save_for_backward(xd, yd, f, g)
                    ctx.weights = (a, b)
                    ctx.eps = eps
                    ctx.ground_cost = ground_cost
                    ctx.report = report
                    return value.to(x.dtype)

                @staticmethod
                def backward(ctx, grad_out):
                    x, y, f, g = ctx.saved_tensors
                    a, b = ctx.weights
                    gx = gy = None
                    if ctx.needs_input_grad[0]:
                        # 2 (a_i x_i - sum_j P_ij y_j), the plan of (F(g), g)
                        gx = grad_x(x, y, g, a, b, eps=ctx.eps,
                                    ground_cost=ctx.ground_cost) * grad_out
                    if ctx.needs_input_grad[1]:
                        # the same with the clouds' roles swapped: the plan of (f, G(f))
                        gy = grad_x(y, x, f, b, a, eps=ctx.eps,
                                    ground_cost=ctx.ground_cost) * grad_out
                    return gx, gy, None, None, None, None, None

            class DivergenceFunction(torch.autograd.Function):
                @staticmethod
                def forward(ctx, x, y, a, b, eps, ground_cost, options):
                    value, gx, gy = sinkhorn_divergence(x.detach(), y.detach(), a, b, eps=eps,
                                                        ground_cost=ground_cost, grads=True,
                                                        **options)
                    ctx.save_for_backward(gx, gy)
                    return value.to(x.dtype)

                @staticmethod
                def backward(ctx, grad_out):
                    gx, gy = ctx.saved_tensors
                    return gx * grad_out, gy * grad_out, None, None, None, None, None

            cls.fn = OTLossFunction
            cls.div = DivergenceFunction
        return cls.fn


class SamplesLoss:
    """Entropic optimal transport loss between two weighted point clouds.

    ``SamplesLoss(eps, n_iters=200, variant="alternating", alpha=0.5, stop_mode="fixed",
    stop_max_iter=20000, stop_tol=1e-6, stop_check_every=5, ground_cost="sqeuclidean")``
    (or "cosine"), ``debias=False`` (True: the debiased divergence
    OT(a, b) - OT(a, a)/2 - OT(b, b)/2 and its gradients); ``loss(x, y, a=None, b=None)``
    returns OT_eps as a 0-d tensor (the dual objective <f,a> + <g,b> - eps (sum P - m_a m_b)
    at the solved potentials) with gradients for x and y; ``loss(x, y, potentials=True)``
    returns the potentials (f, g) in cost units instead. ``last_report`` holds the solve's
    iters_run, converged and final_viol.
    """

    def __init__(self, eps: float = 0.05, n_iters: int = 200, variant: str = "alternating",
                 alpha: float = 0.5, stop_mode: str = "fixed", stop_max_iter: int = 20000,
                 stop_tol: float = 1e-6, stop_check_every: int = 5,
                 ground_cost: str = "sqeuclidean", debias: bool = False):
        self.eps = float(eps)
        self.ground_cost = ground_cost
        self.debias = debias
        self.options = dict(n_iters=n_iters, variant=variant, alpha=alpha, stop_mode=stop_mode,
                            stop_max_iter=stop_max_iter, stop_tol=stop_tol,
                            stop_check_every=stop_check_every)
        self.last_report = None

    def __call__(self, x, y, a=None, b=None, potentials: bool = False):
        if potentials:
            f, g, self.last_report = solve(x.detach(), y.detach(), a, b, eps=self.eps,
                                           ground_cost=self.ground_cost, **self.options)
            return f, g
        fn = _OTLoss.get()
        if self.debias:
            fn = _OTLoss.div
        return fn.apply(x, y, a, b, self.eps, self.ground_cost, self.options)
