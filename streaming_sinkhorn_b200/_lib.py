"""ctypes declarations of the C ABI in include/fs.h (libfs.so, built in-tree).

Loading fails loudly when the library is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfs.so")

FS_MAX_D = 1024

STATUS = {
    0: "FS_OK", 1: "FS_ERR_NULL", 2: "FS_ERR_SHAPE", 3: "FS_ERR_EPS", 4: "FS_ERR_ITERS",
    5: "FS_ERR_NEGATIVE_WEIGHT", 6: "FS_ERR_NONFINITE_INPUT", 7: "FS_ERR_MASS_MISMATCH",
    8: "FS_ERR_ZERO_MASS", 9: "FS_ERR_UNSUPPORTED_D", 10: "FS_ERR_WORKSPACE",
    11: "FS_ERR_TIMEOUT", 12: "FS_ERR_CUDA", 13: "FS_ERR_ALIGNMENT", 14: "FS_ERR_OPTION",
    15: "FS_ERR_DEVICE_MEMORY",
}
STATUS_CODE = {v: k for k, v in STATUS.items()}

# Every function the header declares; the CPU tests check that each one is exported.
EXPORTS = (
    "fs_status_string", "fs_last_cuda_error", "fs_workspace_bytes", "fs_potentials", "fs_cost",
    "fs_grad_x", "fs_marginal_residual", "fs_solve_host_workspace_bytes", "fs_solve_host",
    "fs_timing_enable", "fs_timing_reset", "fs_timing_get", "fs_launch_count",
    "fs_potentials_noalloc", "fs_screening_enable", "fs_solve", "fs_transport_workspace_bytes",
    "fs_transport_apply", "fs_hvp", "fs_divergence_workspace_bytes", "fs_divergence",
    "fs_multiscale_workspace_bytes", "fs_solve_multiscale", "fs_workspace_invalidate",
    "fs_inject_error_word", "fs_check_bounded_wait",
)

VARIANTS = {"alternating": 0, "symmetric": 1}
STOP_MODES = {"fixed": 0, "marginal": 1, "potential": 2}


class fs_problem(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("y", ctypes.c_void_p), ("a", ctypes.c_void_p),
                ("b", ctypes.c_void_p), ("n", ctypes.c_int64), ("m", ctypes.c_int64),
                ("d", ctypes.c_int32), ("eps", ctypes.c_float), ("cost", ctypes.c_int32)]


COSTS = {"sqeuclidean": 0, "cosine": 1}


class fs_solve_options(ctypes.Structure):
    _fields_ = [("n_iters", ctypes.c_int32), ("variant", ctypes.c_int32),
                ("alpha", ctypes.c_float), ("stop_mode", ctypes.c_int32),
                ("stop_max_iter", ctypes.c_int32), ("stop_check_every", ctypes.c_int32),
                ("stop_tol", ctypes.c_double), ("g_init", ctypes.c_void_p)]


class fs_solve_report(ctypes.Structure):
    _fields_ = [("iters_run", ctypes.c_int32), ("converged", ctypes.c_int32),
                ("final_viol", ctypes.c_double)]


class fs_multiscale_options(ctypes.Structure):
    _fields_ = [("cell_points", ctypes.c_int32), ("coarse_iters", ctypes.c_int32),
                ("max_rounds", ctypes.c_int32), ("lift_tol", ctypes.c_double),
                ("lift_shrink", ctypes.c_double)]


class fs_multiscale_report(ctypes.Structure):
    _fields_ = [("rounds", ctypes.c_int32), ("coarse_iters", ctypes.c_int32),
                ("lift_viol", ctypes.c_double), ("fine", fs_solve_report)]


class fs_hvp_options(ctypes.Structure):
    _fields_ = [("cg_max_iter", ctypes.c_int32), ("cg_tol", ctypes.c_double)]


class fs_hvp_report(ctypes.Structure):
    _fields_ = [("cg_iters", ctypes.c_int32), ("cg_rel_residual", ctypes.c_double)]


class fs_timing_entry(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_int64), ("total_ms", ctypes.c_double),
                ("pairs", ctypes.c_double), ("evaluated", ctypes.c_double)]


class fs_timing(ctypes.Structure):
    _fields_ = [("lse_pass", fs_timing_entry), ("grad_pass", fs_timing_entry),
                ("marg_pass", fs_timing_entry), ("combine", fs_timing_entry),
                ("screen", fs_timing_entry)]


_lib = None


def load():
    """The loaded libfs.so with argument types declared. Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m streaming_sinkhorn_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(fs_problem)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    lib.fs_status_string.argtypes = [ctypes.c_int]
    lib.fs_status_string.restype = ctypes.c_char_p
    lib.fs_last_cuda_error.argtypes = []
    lib.fs_last_cuda_error.restype = ctypes.c_char_p
    lib.fs_workspace_bytes.argtypes = [P]
    lib.fs_workspace_bytes.restype = sz
    lib.fs_potentials.argtypes = [P, i32, vp, vp, vp, vp, sz, vp]
    lib.fs_cost.argtypes = [P, vp, vp, vp, vp, sz, vp]
    lib.fs_grad_x.argtypes = [P, vp, vp, vp, sz, vp]
    lib.fs_marginal_residual.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.fs_solve_host_workspace_bytes.argtypes = [P]
    lib.fs_solve_host_workspace_bytes.restype = sz
    lib.fs_solve_host.argtypes = [P, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.fs_solve.argtypes = [P, ctypes.POINTER(fs_solve_options), vp, vp,
                             ctypes.POINTER(fs_solve_report), vp, sz, vp]
    lib.fs_transport_workspace_bytes.argtypes = [P]
    lib.fs_transport_workspace_bytes.restype = sz
    lib.fs_transport_apply.argtypes = [P, vp, vp, i32, i32, vp, vp, vp, sz, vp]
    lib.fs_hvp.argtypes = [P, vp, vp, vp, ctypes.POINTER(fs_hvp_options),
                           ctypes.POINTER(fs_hvp_report), vp, sz, vp]
    lib.fs_multiscale_workspace_bytes.argtypes = [P, i32]
    lib.fs_multiscale_workspace_bytes.restype = sz
    lib.fs_solve_multiscale.argtypes = [P, ctypes.POINTER(fs_solve_options),
                                        ctypes.POINTER(fs_multiscale_options), vp, vp,
                                        ctypes.POINTER(fs_multiscale_report), vp, sz, vp]
    lib.fs_solve_multiscale.restype = ctypes.c_int
    lib.fs_divergence_workspace_bytes.argtypes = [P]
    lib.fs_divergence_workspace_bytes.restype = sz
    lib.fs_divergence.argtypes = [P, ctypes.POINTER(fs_solve_options), vp, vp, vp, vp, sz, vp]
    for fn in (lib.fs_potentials, lib.fs_cost, lib.fs_grad_x, lib.fs_marginal_residual,
               lib.fs_solve_host, lib.fs_solve, lib.fs_transport_apply, lib.fs_hvp,
               lib.fs_divergence):
        fn.restype = ctypes.c_int
    lib.fs_timing_enable.argtypes = [ctypes.c_int]
    lib.fs_timing_enable.restype = None
    lib.fs_screening_enable.argtypes = [ctypes.c_int]
    lib.fs_screening_enable.restype = None
    lib.fs_workspace_invalidate.argtypes = [vp, sz, vp]
    lib.fs_workspace_invalidate.restype = ctypes.c_int
    lib.fs_timing_reset.argtypes = []
    lib.fs_timing_reset.restype = None
    lib.fs_timing_get.argtypes = [ctypes.POINTER(fs_timing)]
    lib.fs_timing_get.restype = None
    lib.fs_potentials_noalloc.argtypes = [P, i32, vp, vp, vp, vp]
    lib.fs_potentials_noalloc.restype = ctypes.c_int
    lib.fs_inject_error_word.argtypes = [ctypes.c_uint]
    lib.fs_inject_error_word.restype = None
    lib.fs_check_bounded_wait.argtypes = [ctypes.c_int64, vp, sz, vp]
    lib.fs_check_bounded_wait.restype = ctypes.c_int
    lib.fs_launch_count.argtypes = []
    lib.fs_launch_count.restype = ctypes.c_int64
    _lib = lib
    return lib
