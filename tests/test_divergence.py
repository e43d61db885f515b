"""The debiased divergence on the GPU (fs_divergence) against the oracle: value and both
gradients under a fixed schedule, zero on equal clouds, and the debiased autograd loss."""
import numpy as np
import pytest

import oracle
import streaming_sinkhorn_b200 as fs
from streaming_sinkhorn_b200 import workloads
from tests.parity_util import assert_grad_close, inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [(300, 257, 2, 0.1), (200, 350, 3, 0.05), (128, 96, 8, 0.5)],
                         ids=lambda s: "n{}-m{}-d{}".format(*s[:3]))
def test_divergence_and_gradients_match_oracle(shape):
    n, m, d, eps = shape
    w = workloads.random_small(n, m, d, seed=n + m, eps=eps, n_iters=15)
    x, y, a, b = inputs(w)
    value, gx, gy = fs.sinkhorn_divergence(x, y, a, b, eps=w.eps, n_iters=w.n_iters, grads=True)
    ref, rgx, rgy = oracle.divergence(w.x, w.y, w.a, w.b, w.eps, grads=True, n_iters=w.n_iters)
    # S is a difference of three duals of size ~ OT(x, y): compare on that scale
    scale = abs(oracle.divergence(w.x, w.y, w.a, w.b, w.eps, n_iters=w.n_iters)) + 1e-3
    assert abs(float(value) - ref) <= 1e-4 * max(scale, 1.0)
    assert_grad_close(gx.cpu().numpy(), rgx)
    assert_grad_close(gy.cpu().numpy(), rgy)


def test_divergence_of_equal_clouds_is_zero():
    w = workloads.random_small(200, 200, 3, seed=8, eps=0.1, n_iters=10)
    x, _, a, _ = inputs(w)
    value, gx, gy = fs.sinkhorn_divergence(x, x, a, a, eps=w.eps, n_iters=w.n_iters, grads=True)
    assert abs(float(value)) < 1e-5
    assert np.abs(gx.cpu().numpy()).max() < 1e-4 * np.abs(w.x).max()


def test_debiased_loss_backward():
    w = workloads.random_small(150, 130, 2, seed=9, eps=0.2, n_iters=20)
    x, y, a, b = inputs(w)
    x = x.clone().requires_grad_(True)
    y = y.clone().requires_grad_(True)
    loss = fs.SamplesLoss(eps=w.eps, n_iters=w.n_iters, debias=True)
    (2.0 * loss(x, y, a, b)).backward()
    _, rgx, rgy = oracle.divergence(w.x, w.y, w.a, w.b, w.eps, grads=True, n_iters=w.n_iters)
    assert_grad_close(x.grad.cpu().numpy() / 2.0, rgx)
    assert_grad_close(y.grad.cpu().numpy() / 2.0, rgy)
