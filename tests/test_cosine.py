"""The cosine cost on the GPU against the oracle: potentials, cost and gradient, on the FMA
and the tensor-core paths, and a zero point rejected."""
import numpy as np
import pytest

import oracle
import streaming_sinkhorn_b200 as fs
from streaming_sinkhorn_b200 import workloads
from tests.parity_util import assert_cost_close, assert_grad_close, assert_potential_close, inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [(300, 257, 3, 0.05), (500, 400, 16, 0.1), (200, 240, 64, 0.2)],
                         ids=lambda s: "n{}-m{}-d{}".format(*s[:3]))
def test_cosine_potentials_cost_and_gradient(shape):
    n, m, d, eps = shape
    w = workloads.random_small(n, m, d, seed=n + d, eps=eps, n_iters=12)
    x, y, a, b = inputs(w)
    f, g = fs.potentials(x, y, a, b, eps=w.eps, n_iters=w.n_iters, ground_cost="cosine")
    xs, ys = oracle.cosine_inputs(w.x, w.y)
    fr, gr = oracle.potentials(xs, ys, w.a, w.b, w.eps, w.n_iters)
    rel = 5e-3 if d >= 32 else 1e-4
    assert_potential_close(f.cpu().numpy(), fr, "f", rel=rel)
    assert_potential_close(g.cpu().numpy(), gr, "g", rel=rel)
    c = fs.cost(x, y, f, g, a, b, eps=w.eps, ground_cost="cosine").item()
    assert_cost_close(c, oracle.cost(xs, ys, w.a, w.b, w.eps, f.cpu().numpy(), g.cpu().numpy()),
                      rel=rel)
    gx = fs.grad_x(x, y, g, a, b, eps=w.eps, ground_cost="cosine").cpu().numpy()
    assert_grad_close(gx, oracle.grad_x_cosine(w.x, w.y, w.a, w.b, w.eps, g.cpu().numpy()),
                      rel=5e-3 if d >= 32 else 1e-4)


def test_cosine_zero_point_is_rejected():
    w = workloads.random_small(50, 40, 3, seed=1, eps=0.1)
    w.x[7] = 0.0
    x, y, a, b = inputs(w)
    with pytest.raises(fs.FsError, match="NONFINITE"):
        fs.potentials(x, y, a, b, eps=w.eps, n_iters=2, ground_cost="cosine")


def test_cosine_loss_gradient():
    w = workloads.random_small(150, 120, 8, seed=3, eps=0.1, n_iters=20)
    x, y, a, b = inputs(w)
    x = x.clone().requires_grad_(True)
    loss = fs.SamplesLoss(eps=w.eps, n_iters=w.n_iters, ground_cost="cosine")
    loss(x, y, a, b).backward()
    xs, ys = oracle.cosine_inputs(w.x, w.y)
    _, gr = oracle.potentials(xs, ys, w.a, w.b, w.eps, w.n_iters)
    assert_grad_close(x.grad.cpu().numpy(), oracle.grad_x_cosine(w.x, w.y, w.a, w.b, w.eps, gr))
    # the gradient is orthogonal to each point
    gx = x.grad.cpu().numpy().astype(np.float64)
    assert np.abs((gx * w.x).sum(1)).max() < 1e-4 * np.abs(gx).max() * np.abs(w.x).max()
