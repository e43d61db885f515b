"""fs_potentials_noalloc: the solve for callers that cannot allocate device memory (for
example, an application whose device memory is owned by its own pool allocator, or a
latency-critical loop that must avoid the device synchronisation cudaMalloc/cudaFree can
cause). Its scratch space is a fixed array in device global memory owned by the library.

The GPU test calls the entry point through the C ABI, passing only inputs and outputs,
and checks two calls in a row against fs_potentials (which takes a caller workspace)
within the potential tolerance the other parity tests use. The file is named to be
collected last, so a stop-at-first-failure run has run every other test before it.
"""
import ctypes

import numpy as np
import pytest

from streaming_sinkhorn_b200 import _lib, workloads

FAKE = 0x7F0000000000  # never dereferenced: the call must refuse before touching memory


def test_rejects_problems_larger_than_the_static_scratch():
    """Host-side refusal, no device work: safe without a GPU."""
    lib = _lib.load()
    limit = 20 << 20
    p = _lib.fs_problem(FAKE, FAKE, None, None, 2_000_000, 2_000_000, 3, 0.1)
    assert lib.fs_workspace_bytes(ctypes.byref(p)) > limit
    code = lib.fs_potentials_noalloc(ctypes.byref(p), 5, None, FAKE, FAKE, None)
    assert _lib.STATUS[code] == "FS_ERR_WORKSPACE"
    bad = _lib.fs_problem(FAKE, FAKE, None, None, 0, 10, 3, 0.1)
    assert _lib.STATUS[lib.fs_potentials_noalloc(ctypes.byref(bad), 5, None, FAKE, FAKE,
                                                 None)] == "FS_ERR_SHAPE"
    assert _lib.STATUS[lib.fs_potentials_noalloc(None, 5, None, FAKE, FAKE, None)] == "FS_ERR_NULL"


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point():
    import torch
    import streaming_sinkhorn_b200 as fs
    from tests.parity_util import assert_potential_close

    w = workloads.random_small(3000, 2500, 3, seed=21, eps=0.05, zero_frac=0.05, n_iters=10)
    dev = lambda v: torch.from_numpy(v).cuda()  # noqa: E731
    x, y, a, b = dev(w.x), dev(w.y), dev(w.a), dev(w.b)
    f_ref, g_ref = fs.potentials(x, y, a, b, eps=w.eps, n_iters=w.n_iters)
    f_ref, g_ref = f_ref.cpu().numpy(), g_ref.cpu().numpy()

    lib = _lib.load()
    p = _lib.fs_problem(x.data_ptr(), y.data_ptr(), a.data_ptr(), b.data_ptr(), w.n, w.m, w.d,
                        w.eps)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        f = torch.full((w.n,), float("nan"), device="cuda")
        g = torch.full((w.m,), float("nan"), device="cuda")
        code = lib.fs_potentials_noalloc(ctypes.byref(p), w.n_iters, None, f.data_ptr(),
                                         g.data_ptr(), stream)
        assert _lib.STATUS[code] == "FS_OK", lib.fs_last_cuda_error()
        torch.cuda.synchronize()
        assert np.isfinite(f.cpu().numpy()).all() and np.isfinite(g.cpu().numpy()).all()
        assert_potential_close(f.cpu().numpy(), f_ref, "f")
        assert_potential_close(g.cpu().numpy(), g_ref, "g")


@pytest.mark.gpu
def test_documented_size_fits_the_static_scratch():
    """The header promises that every d = 3 problem with n, m <= 80000 fits; the workspace
    depends on the device's occupancy, so this is checked on the GPU."""
    lib = _lib.load()
    for n, m in ((80000, 80000), (80000, 1), (1, 80000), (65536, 80000)):
        p = _lib.fs_problem(FAKE, FAKE, None, None, n, m, 3, 0.1)
        assert lib.fs_workspace_bytes(ctypes.byref(p)) <= 20 << 20, (n, m)
