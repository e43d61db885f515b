"""The error path on the GPU: a kernel whose bounded wait expires sets the call's device
error word and the call returns FS_ERR_TIMEOUT instead of results (SinkSLOT README, "Tensor
Contract": invalid states raise rather than return wrong values).

No GPU is faulted, trapped or hung here. The bounded-wait check waits, with a 50 ms limit,
on a barrier nothing arrives at and with no copy in flight; the injection test ORs a bit
into the error word from a kernel after the passes. Both check that the status reaches the
caller and that the next call on the same workspace is correct again.
"""
import ctypes
import time

import numpy as np
import pytest

import oracle
from streaming_sinkhorn_b200 import _lib, workloads
from tests.parity_util import assert_potential_close

pytestmark = pytest.mark.gpu


def _setup(n=600, m=500, d=3, seed=5):
    import torch
    w = workloads.random_small(n, m, d, seed=seed, eps=0.1, zero_frac=0.05, n_iters=7)
    dev = lambda v: torch.from_numpy(v).cuda()  # noqa: E731
    x, y, a, b = dev(w.x), dev(w.y), dev(w.a), dev(w.b)
    lib = _lib.load()
    p = _lib.fs_problem(x.data_ptr(), y.data_ptr(), a.data_ptr(), b.data_ptr(), w.n, w.m, w.d,
                        w.eps)
    need = lib.fs_workspace_bytes(ctypes.byref(p))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    f = torch.empty(w.n, device="cuda")
    g = torch.empty(w.m, device="cuda")
    keep = (x, y, a, b)
    return w, lib, p, ws, need, f, g, keep


def _solve(lib, p, w, ws, need, f, g):
    import torch
    stream = torch.cuda.current_stream().cuda_stream
    code = lib.fs_potentials(ctypes.byref(p), w.n_iters, None, f.data_ptr(), g.data_ptr(),
                             ws.data_ptr(), need, stream)
    torch.cuda.synchronize()
    return _lib.STATUS[code]


def test_bounded_wait_expires_and_the_context_stays_usable():
    import torch
    w, lib, p, ws, need, f, g, _keep = _setup()
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    code = lib.fs_check_bounded_wait(50_000_000, ws.data_ptr(), need, stream)
    dt = time.perf_counter() - t0
    assert _lib.STATUS[code] == "FS_ERR_TIMEOUT"
    assert lib.fs_status_string(code).decode().startswith("FS_ERR_TIMEOUT")
    assert 0.04 <= dt < 5.0, dt
    # out-of-range limits are refused before any device work
    assert _lib.STATUS[lib.fs_check_bounded_wait(10, ws.data_ptr(), need, stream)] == "FS_ERR_OPTION"
    assert _lib.STATUS[lib.fs_check_bounded_wait(50_000_000, ws.data_ptr(), 64,
                                                 stream)] == "FS_ERR_WORKSPACE"
    # the same workspace and context then give a correct solve
    assert _solve(lib, p, w, ws, need, f, g) == "FS_OK"
    fr, gr = oracle.potentials(w.x, w.y, w.a, w.b, w.eps, w.n_iters)
    assert_potential_close(f.cpu().numpy(), fr, "f")
    assert_potential_close(g.cpu().numpy(), gr, "g")


def test_injected_error_word_is_reported_once():
    import streaming_sinkhorn_b200 as fs
    w, lib, p, ws, need, f, g, (x, y, a, b) = _setup(seed=6)
    try:
        lib.fs_inject_error_word(1)
        assert _solve(lib, p, w, ws, need, f, g) == "FS_ERR_TIMEOUT"
        # disarmed by that call: the next call on the same workspace is correct
        assert _solve(lib, p, w, ws, need, f, g) == "FS_OK"
        fr, gr = oracle.potentials(w.x, w.y, w.a, w.b, w.eps, w.n_iters)
        assert_potential_close(f.cpu().numpy(), fr, "f")
        assert_potential_close(g.cpu().numpy(), gr, "g")
        # through the Python layer the status becomes an exception naming it
        lib.fs_inject_error_word(4)
        with pytest.raises(fs.FsError) as ei:
            fs.grad_x(x, y, g, a, b, eps=w.eps)
        assert ei.value.status == "FS_ERR_TIMEOUT"
        gx = fs.grad_x(x, y, g, a, b, eps=w.eps).cpu().numpy()
        gxr = oracle.grad_x(w.x, w.y, w.a, w.b, w.eps, g.cpu().numpy())
        assert np.abs(gx - gxr).max() <= 1e-4 * np.abs(gxr).max()
    finally:
        lib.fs_inject_error_word(0)
