"""The C ABI on the CPU: the library loads, exports every declared entry point, and
rejects bad arguments before touching a device. No GPU is needed or used here."""
import ctypes
import os
import re

import numpy as np
import pytest

from streaming_sinkhorn_b200 import _lib
import streaming_sinkhorn_b200 as fs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fs.h")

# A fake, 256-byte aligned "device" address: only ever compared, never dereferenced.
FAKE = 0x7F0000000000
BIG = 1 << 40


def declared_functions():
    text = open(HEADER).read()
    return set(re.findall(r"FS_API\s+[\w\s\*]+?\b(fs_\w+)\s*\(", text))


def test_header_declares_the_exported_set():
    assert declared_functions() == set(_lib.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings():
    lib = _lib.load()
    for code, name in _lib.STATUS.items():
        s = lib.fs_status_string(code).decode()
        assert s.startswith(name)
    assert lib.fs_status_string(999).decode() == "unknown fs_status"


def prob(n=10, m=12, d=3, eps=0.1, x=FAKE, y=FAKE + 4096, a=None, b=None):
    return _lib.fs_problem(x, y, a, b, n, m, d, eps)


def test_workspace_bytes():
    lib = _lib.load()
    small = lib.fs_workspace_bytes(ctypes.byref(prob()))
    assert small > 0 and small % 256 == 0
    big = lib.fs_workspace_bytes(ctypes.byref(prob(n=1 << 20, m=1 << 20)))
    assert big > small
    # packed keys alone: 2 clouds x (2^19 pairs x 8 floats x 4 B) = 32 MiB for d = 3
    assert big >= 2 * (1 << 19) * 8 * 4
    for bad in (prob(n=0), prob(m=0), prob(d=0), prob(d=1025)):
        assert lib.fs_workspace_bytes(ctypes.byref(bad)) == 0
    assert lib.fs_workspace_bytes(None) == 0


@pytest.mark.parametrize("p,expect", [
    (None, "FS_ERR_NULL"),
    (prob(n=0), "FS_ERR_SHAPE"),
    (prob(m=-3), "FS_ERR_SHAPE"),
    (prob(d=0), "FS_ERR_SHAPE"),
    (prob(d=1025), "FS_ERR_UNSUPPORTED_D"),
    (prob(eps=0.0), "FS_ERR_EPS"),
    (prob(eps=-1.0), "FS_ERR_EPS"),
    (prob(eps=float("nan")), "FS_ERR_EPS"),
    (prob(eps=float("inf")), "FS_ERR_EPS"),
    (prob(x=None), "FS_ERR_NULL"),
    (prob(y=None), "FS_ERR_NULL"),
    (prob(x=FAKE + 2), "FS_ERR_ALIGNMENT"),
    (prob(a=FAKE + 1), "FS_ERR_ALIGNMENT"),
])
def test_host_side_argument_errors(p, expect):
    lib = _lib.load()
    ref = None if p is None else ctypes.byref(p)
    code = lib.fs_potentials(ref, 3, None, FAKE, FAKE, FAKE, BIG, None)
    assert _lib.STATUS[code] == expect
    assert _lib.STATUS[lib.fs_grad_x(ref, FAKE, FAKE, FAKE, BIG, None)] == expect
    assert _lib.STATUS[lib.fs_cost(ref, FAKE, FAKE, FAKE, FAKE, BIG, None)] == expect
    assert _lib.STATUS[lib.fs_marginal_residual(ref, FAKE, FAKE, FAKE, None, None, FAKE, BIG,
                                                None)] == expect


def test_workspace_and_output_errors():
    lib = _lib.load()
    p = ctypes.byref(prob())
    need = lib.fs_workspace_bytes(p)
    st = lambda c: _lib.STATUS[c]  # noqa: E731
    assert st(lib.fs_potentials(p, 3, None, FAKE, FAKE, None, BIG, None)) == "FS_ERR_WORKSPACE"
    assert st(lib.fs_potentials(p, 3, None, FAKE, FAKE, FAKE + 8, BIG, None)) == "FS_ERR_WORKSPACE"
    assert st(lib.fs_potentials(p, 3, None, FAKE, FAKE, FAKE, need - 1, None)) == "FS_ERR_WORKSPACE"
    assert st(lib.fs_potentials(p, 3, None, None, FAKE, FAKE, need, None)) == "FS_ERR_NULL"
    assert st(lib.fs_potentials(p, 3, None, FAKE + 1, FAKE, FAKE, need, None)) == "FS_ERR_ALIGNMENT"
    assert st(lib.fs_potentials(p, 0, None, FAKE, FAKE, FAKE, need, None)) == "FS_ERR_ITERS"
    assert st(lib.fs_potentials(p, -5, None, FAKE, FAKE, FAKE, need, None)) == "FS_ERR_ITERS"
    assert st(lib.fs_grad_x(p, None, FAKE, FAKE, need, None)) == "FS_ERR_NULL"
    assert st(lib.fs_cost(p, FAKE, FAKE, FAKE + 4, FAKE, need, None)) == "FS_ERR_ALIGNMENT"
    assert st(lib.fs_marginal_residual(p, FAKE, FAKE, None, None, None, FAKE, need,
                                       None)) == "FS_ERR_NULL"


def test_solve_host_argument_errors():
    lib = _lib.load()
    x = np.zeros((4, 2), np.float32)
    hp = _lib.fs_problem(x.ctypes.data, x.ctypes.data, None, None, 4, 4, 2, 0.1)
    need = lib.fs_solve_host_workspace_bytes(ctypes.byref(hp))
    assert need > lib.fs_workspace_bytes(ctypes.byref(hp))
    f = np.zeros(4, np.float32)
    st = lambda c: _lib.STATUS[c]  # noqa: E731
    assert st(lib.fs_solve_host(None, 1, f.ctypes.data, f.ctypes.data, None, None, None, FAKE,
                                need, None)) == "FS_ERR_NULL"
    assert st(lib.fs_solve_host(ctypes.byref(hp), 0, f.ctypes.data, f.ctypes.data, None, None,
                                None, FAKE, need, None)) == "FS_ERR_ITERS"
    assert st(lib.fs_solve_host(ctypes.byref(hp), 1, f.ctypes.data, f.ctypes.data, None, None,
                                None, FAKE, need - 256, None)) == "FS_ERR_WORKSPACE"


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="passes fake device pointers: only meaningful without a GPU")
def test_without_a_device_the_call_fails_loudly():
    """Valid host-side arguments but no CUDA device: FS_ERR_CUDA, never a CPU fallback."""
    lib = _lib.load()
    p = ctypes.byref(prob())
    need = lib.fs_workspace_bytes(p)
    code = lib.fs_potentials(p, 2, None, FAKE, FAKE, FAKE, need, None)
    assert _lib.STATUS[code] == "FS_ERR_CUDA"
    assert lib.fs_last_cuda_error().decode() != ""


def test_python_binding_rejects_cpu_and_float64():
    import torch
    x = torch.zeros(5, 2)
    with pytest.raises(ValueError, match="CUDA"):
        fs.potentials(x, x, eps=0.1, n_iters=1)
    with pytest.raises(ValueError, match="float64"):
        fs.potentials(x.double(), x.double(), eps=0.1, n_iters=1)
    with pytest.raises(ValueError, match="float64"):
        fs.solve_host(x.double().numpy(), x.double().numpy(), eps=0.1, n_iters=1)


def test_timing_api_roundtrip():
    fs.timing_enable(True)
    fs.timing_reset()
    t = fs.timing_get()
    assert set(t) == {"lse_pass", "grad_pass", "marg_pass", "combine", "screen"}
    assert all(v["launches"] == 0 for v in t.values())
    fs.timing_enable(False)


def test_solve_option_errors():
    lib = _lib.load()
    p = ctypes.byref(prob())
    need = lib.fs_workspace_bytes(p)
    st = lambda c: _lib.STATUS[c]  # noqa: E731

    def opts(**kw):
        o = dict(n_iters=5, variant=0, alpha=0.5, stop_mode=0, stop_max_iter=100,
                 stop_check_every=5, stop_tol=1e-6, g_init=None)
        o.update(kw)
        return _lib.fs_solve_options(o["n_iters"], o["variant"], o["alpha"], o["stop_mode"],
                                     o["stop_max_iter"], o["stop_check_every"], o["stop_tol"],
                                     o["g_init"])

    rep = _lib.fs_solve_report()
    call = lambda o: st(lib.fs_solve(p, ctypes.byref(o), FAKE, FAKE, ctypes.byref(rep), FAKE,  # noqa: E731
                                     need, None))
    assert st(lib.fs_solve(p, None, FAKE, FAKE, None, FAKE, need, None)) == "FS_ERR_NULL"
    assert call(opts(n_iters=0)) == "FS_ERR_ITERS"
    assert call(opts(variant=2)) == "FS_ERR_OPTION"
    assert call(opts(variant=1, alpha=0.0)) == "FS_ERR_OPTION"
    assert call(opts(variant=1, alpha=1.5)) == "FS_ERR_OPTION"
    assert call(opts(stop_mode=3)) == "FS_ERR_OPTION"
    assert call(opts(stop_mode=1, stop_max_iter=0)) == "FS_ERR_OPTION"
    assert call(opts(stop_mode=2, stop_check_every=0)) == "FS_ERR_OPTION"
    assert call(opts(stop_mode=1, stop_tol=-1.0)) == "FS_ERR_OPTION"
    assert call(opts(stop_mode=1, stop_tol=float("nan"))) == "FS_ERR_OPTION"
    assert st(lib.fs_solve(p, ctypes.byref(opts()), FAKE + 2, FAKE, None, FAKE, need,
                           None)) == "FS_ERR_ALIGNMENT"


def test_transport_and_hvp_argument_errors():
    lib = _lib.load()
    p = ctypes.byref(prob())
    base = lib.fs_workspace_bytes(p)
    need = lib.fs_transport_workspace_bytes(p)
    assert need > base and need % 256 == 0
    assert lib.fs_transport_workspace_bytes(ctypes.byref(prob(d=17))) > 0  # tensor-core path
    assert lib.fs_transport_workspace_bytes(ctypes.byref(prob(d=1025))) == 0
    assert lib.fs_transport_workspace_bytes(None) == 0
    st = lambda c: _lib.STATUS[c]  # noqa: E731
    ta = lambda *a: st(lib.fs_transport_apply(*a))  # noqa: E731
    assert ta(p, FAKE, FAKE, 0, 0, FAKE, FAKE, FAKE, need, None) == "FS_ERR_OPTION"
    assert ta(p, FAKE, FAKE, 2, 3, FAKE, FAKE, FAKE, need, None) == "FS_ERR_OPTION"
    assert ta(p, None, FAKE, 0, 3, FAKE, FAKE, FAKE, need, None) == "FS_ERR_NULL"
    assert ta(p, FAKE, FAKE, 0, 3, FAKE + 2, FAKE, FAKE, need, None) == "FS_ERR_ALIGNMENT"
    assert ta(p, FAKE, FAKE, 0, 3, FAKE, FAKE, FAKE, need - 256, None) == "FS_ERR_WORKSPACE"
    too_wide = ctypes.byref(prob(d=1025))
    assert ta(too_wide, FAKE, FAKE, 0, 3, FAKE, FAKE, FAKE, BIG, None) == "FS_ERR_UNSUPPORTED_D"
    hv = lambda *a: st(lib.fs_hvp(*a))  # noqa: E731
    bad_iter = _lib.fs_hvp_options(0, 1e-6)
    bad_tol = _lib.fs_hvp_options(10, -1.0)
    assert hv(p, FAKE, FAKE, FAKE, ctypes.byref(bad_iter), None, FAKE, need, None) == "FS_ERR_OPTION"
    assert hv(p, FAKE, FAKE, FAKE, ctypes.byref(bad_tol), None, FAKE, need, None) == "FS_ERR_OPTION"
    assert hv(p, FAKE, None, FAKE, None, None, FAKE, need, None) == "FS_ERR_NULL"
    assert hv(too_wide, FAKE, FAKE, FAKE, None, None, FAKE, BIG, None) == "FS_ERR_UNSUPPORTED_D"
    # the HVP's difference pass has no wide form: d > 64 is refused before any device work
    hvp_wide = ctypes.byref(prob(d=65))
    assert hv(hvp_wide, FAKE, FAKE, FAKE, None, None, FAKE, BIG, None) == "FS_ERR_UNSUPPORTED_D"


def test_divergence_argument_errors():
    lib = _lib.load()
    p = ctypes.byref(prob())
    need = lib.fs_divergence_workspace_bytes(p)
    assert need > lib.fs_workspace_bytes(p)
    assert lib.fs_divergence_workspace_bytes(ctypes.byref(prob(d=1025))) == 0
    st = lambda c: _lib.STATUS[c]  # noqa: E731
    o = _lib.fs_solve_options(5, 0, 0.5, 0, 100, 5, 1e-6, None)
    assert st(lib.fs_divergence(p, None, FAKE, None, None, FAKE, need, None)) == "FS_ERR_NULL"
    assert st(lib.fs_divergence(p, ctypes.byref(o), None, None, None, FAKE, need, None)) == "FS_ERR_NULL"
    assert st(lib.fs_divergence(p, ctypes.byref(o), FAKE + 4, None, None, FAKE, need,
                                None)) == "FS_ERR_ALIGNMENT"
    assert st(lib.fs_divergence(p, ctypes.byref(o), FAKE, None, None, FAKE, need - 256,
                                None)) == "FS_ERR_WORKSPACE"
    assert st(lib.fs_divergence(ctypes.byref(prob(n=0)), ctypes.byref(o), FAKE, None, None, FAKE,
                                need, None)) == "FS_ERR_SHAPE"


def test_multiscale_argument_errors():
    lib = _lib.load()
    p = ctypes.byref(prob())
    need = lib.fs_multiscale_workspace_bytes(p, 32)
    assert need > lib.fs_workspace_bytes(p)
    assert lib.fs_multiscale_workspace_bytes(ctypes.byref(prob(d=17)), 32) == 0
    assert lib.fs_multiscale_workspace_bytes(p, 0) == 0
    assert lib.fs_multiscale_workspace_bytes(p, 257) == 0
    st = lambda c: _lib.STATUS[c]  # noqa: E731
    o = _lib.fs_solve_options(5, 0, 0.5, 0, 100, 5, 1e-6, None)
    call = lambda mo, ws=need: st(lib.fs_solve_multiscale(  # noqa: E731
        p, ctypes.byref(o), ctypes.byref(mo), FAKE, FAKE, None, FAKE, ws, None))
    assert call(_lib.fs_multiscale_options(32, 0, 4, 0.0, 0.5)) == "FS_ERR_OPTION"
    assert call(_lib.fs_multiscale_options(32, 5, 0, 0.0, 0.5)) == "FS_ERR_OPTION"
    assert call(_lib.fs_multiscale_options(32, 5, 4, -1.0, 0.5)) == "FS_ERR_OPTION"
    assert call(_lib.fs_multiscale_options(32, 5, 4, 0.0, 0.0)) == "FS_ERR_OPTION"
    assert call(_lib.fs_multiscale_options(0, 5, 4, 0.0, 0.5)) == "FS_ERR_OPTION"
    assert call(_lib.fs_multiscale_options(300, 5, 4, 0.0, 0.5)) == "FS_ERR_OPTION"
    assert call(_lib.fs_multiscale_options(32, 5, 4, 0.0, 0.5), need - 256) == "FS_ERR_WORKSPACE"
    cos = _lib.fs_problem(FAKE, FAKE + 4096, None, None, 10, 12, 3, 0.1, 1)
    assert st(lib.fs_solve_multiscale(ctypes.byref(cos), ctypes.byref(o),
                                      ctypes.byref(_lib.fs_multiscale_options(32, 5, 4, 0.0, 0.5)),
                                      FAKE, FAKE, None, FAKE, BIG, None)) == "FS_ERR_OPTION"


def test_workspace_invalidate_argument_errors():
    """Rejected before any CUDA call: no workspace, a misaligned one, one too small to hold
    the scalar block."""
    lib = _lib.load()
    code = _lib.STATUS_CODE["FS_ERR_WORKSPACE"]
    assert lib.fs_workspace_invalidate(None, 4096, None) == code
    assert lib.fs_workspace_invalidate(FAKE + 16, 4096, None) == code
    assert lib.fs_workspace_invalidate(FAKE, 1024, None) == code
