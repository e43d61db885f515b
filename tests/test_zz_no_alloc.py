"""fs_potentials_noalloc: the solve for callers that cannot allocate device memory (for
example, an application whose device memory is owned by its own pool allocator, or a
latency-critical loop that must avoid the device synchronisation cudaMalloc/cudaFree can
cause). Its scratch space is a fixed array in device global memory owned by the library.

The GPU test calls the entry point through the C ABI, passing only inputs and outputs, and
checks it against fs_potentials (which takes a caller workspace) within the potential
tolerance the other parity tests use: two calls in a row on one problem, then calls on a
problem of another layout (d = 64, the tensor-core path, which clears the array's sort
record) and of another size, then the first problem again, since every call inherits what
the previous one left in the shared array. A warm call must not change the device's free
memory. The file is named to be collected last, so a stop-at-first-failure run has run
every other test before it.
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


class _Case:
    """One problem on the device, with fs_potentials' result as the reference."""

    def __init__(self, n, m, d, seed, eps):
        import torch
        import streaming_sinkhorn_b200 as fs
        self.w = workloads.random_small(n, m, d, seed=seed, eps=eps, zero_frac=0.05, n_iters=10)
        dev = lambda v: torch.from_numpy(v).cuda()  # noqa: E731
        w = self.w
        self.t = (dev(w.x), dev(w.y), dev(w.a), dev(w.b))
        x, y, a, b = self.t
        f_ref, g_ref = fs.potentials(x, y, a, b, eps=w.eps, n_iters=w.n_iters)
        self.f_ref, self.g_ref = f_ref.cpu().numpy(), g_ref.cpu().numpy()
        self.p = _lib.fs_problem(x.data_ptr(), y.data_ptr(), a.data_ptr(), b.data_ptr(), w.n,
                                 w.m, w.d, w.eps)
        self.f = torch.empty(w.n, device="cuda")
        self.g = torch.empty(w.m, device="cuda")

    def call_noalloc(self, lib):
        import torch
        self.f.fill_(float("nan"))
        self.g.fill_(float("nan"))
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream().cuda_stream
        code = lib.fs_potentials_noalloc(ctypes.byref(self.p), self.w.n_iters, None,
                                         self.f.data_ptr(), self.g.data_ptr(), stream)
        torch.cuda.synchronize()
        return _lib.STATUS[code]

    def check(self):
        from tests.parity_util import assert_potential_close
        f, g = self.f.cpu().numpy(), self.g.cpu().numpy()
        assert np.isfinite(f).all() and np.isfinite(g).all()
        assert_potential_close(f, self.f_ref, "f")
        assert_potential_close(g, self.g_ref, "g")


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point():
    import torch

    lib = _lib.load()
    first = _Case(3000, 2500, 3, seed=21, eps=0.05)
    wide = _Case(700, 900, 64, seed=22, eps=4.0)
    other = _Case(1700, 2100, 3, seed=23, eps=0.05)
    for _ in range(2):  # two calls in a row on one problem
        assert first.call_noalloc(lib) == "FS_OK", lib.fs_last_cuda_error()
        first.check()
    # The module holding the array is loaded now: a warm call commits no device memory.
    free0, _ = torch.cuda.mem_get_info()
    assert wide.call_noalloc(lib) == "FS_OK", lib.fs_last_cuda_error()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)
    wide.check()
    assert other.call_noalloc(lib) == "FS_OK", lib.fs_last_cuda_error()
    other.check()
    assert first.call_noalloc(lib) == "FS_OK", lib.fs_last_cuda_error()
    first.check()


@pytest.mark.gpu
def test_documented_size_fits_the_static_scratch():
    """The header promises that every d = 3 problem with n, m <= 80000 fits; the workspace
    depends on the device's occupancy, so this is checked on the GPU."""
    lib = _lib.load()
    for n, m in ((80000, 80000), (80000, 1), (1, 80000), (65536, 80000)):
        p = _lib.fs_problem(FAKE, FAKE, None, None, n, m, 3, 0.1)
        assert lib.fs_workspace_bytes(ctypes.byref(p)) <= 20 << 20, (n, m)
