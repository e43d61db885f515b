"""The autograd loss (SamplesLoss): its value is the dual objective of the solved
potentials, its gradients for x and y are the oracle's envelope gradients, and gradient
descent through it lowers the loss."""
import numpy as np
import pytest
import torch

import oracle
import streaming_sinkhorn_b200 as fs
from streaming_sinkhorn_b200 import workloads
from tests.parity_util import assert_grad_close, inputs

pytestmark = pytest.mark.gpu


def test_value_and_gradients_match_oracle():
    w = workloads.random_small(300, 250, 3, seed=4, eps=0.2, n_iters=30)
    x, y, a, b = inputs(w)
    x = x.clone().requires_grad_(True)
    y = y.clone().requires_grad_(True)
    loss = fs.SamplesLoss(eps=w.eps, n_iters=w.n_iters)
    value = loss(x, y, a, b)
    (3.0 * value).backward()
    f, g = oracle.potentials(w.x, w.y, w.a, w.b, w.eps, w.n_iters)
    assert float(value.detach()) == pytest.approx(oracle.cost(w.x, w.y, w.a, w.b, w.eps, f, g),
                                                rel=1e-4)
    assert_grad_close(x.grad.cpu().numpy() / 3.0, oracle.grad_x(w.x, w.y, w.a, w.b, w.eps, g))
    # the gradient for y: the same formula with the clouds' roles swapped, plan of (f, G(f))
    assert_grad_close(y.grad.cpu().numpy() / 3.0, oracle.grad_x(w.y, w.x, w.b, w.a, w.eps, f))
    assert loss.last_report is None  # set only by the potentials form


def test_potentials_form_and_report():
    w = workloads.random_small(120, 100, 2, seed=5, eps=0.3, n_iters=10)
    x, y, a, b = inputs(w)
    loss = fs.SamplesLoss(eps=w.eps, stop_mode="marginal", stop_tol=1e-6, stop_check_every=5)
    f, g = loss(x, y, a, b, potentials=True)
    assert f.shape == (120,) and g.shape == (100,)
    assert loss.last_report["converged"] is True


def test_gradient_descent_lowers_the_loss():
    w = workloads.gaussian_shifted(n=500, d=2, shift=3.0, seed=0, eps=0.1, n_iters=50)
    x, y, _, _ = inputs(w)
    x = x.clone().requires_grad_(True)
    loss = fs.SamplesLoss(eps=w.eps, n_iters=w.n_iters)
    values = []
    for _ in range(5):
        value = loss(x, y)
        values.append(float(value.detach()))
        (gx,) = torch.autograd.grad(value, [x])
        with torch.no_grad():
            x -= 0.25 * gx / (2.0 / w.n)  # a step of size 0.25 on each point
    assert all(v1 < v0 for v0, v1 in zip(values, values[1:])), values
