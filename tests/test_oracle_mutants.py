"""Plant plausible mistakes in copies of the oracle and check that the pins catch each.

Each mutant is a one-line edit of ``oracle/oracle.c`` (a dropped term, a flipped sign,
a transposed operand, a wrong initial value), compiled into a temporary library on the
CPU. The pin suite of ``test_oracle_pins.py`` is then run against it; at least one pin
must fail. The real oracle is never modified.
"""
import ctypes
import inspect
import os
import subprocess

import numpy as np
import pytest

import oracle
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "dropped_log_weight": ("z[j] = (pot_q[j] - c) / eps + log(wq[j]);",
                           "z[j] = (pot_q[j] - c) / eps;"),
    "potential_sign": ("z[j] = (pot_q[j] - c) / eps", "z[j] = (-pot_q[j] - c) / eps"),
    "cost_sign": ("z[j] = (pot_q[j] - c) / eps", "z[j] = (pot_q[j] + c) / eps"),
    "output_sign": ("out[k] = -eps * (zmax + log(s));", "out[k] = eps * (zmax + log(s));"),
    "dropped_shift": ("out[k] = -eps * (zmax + log(s));", "out[k] = -eps * log(s);"),
    "abs_instead_of_square": ("s += t * t;", "s += fabs(t);"),
    "grad_transposed_operand": ("acc[c] += p * y[j * d + c];", "acc[c] += p * x[i * d + c];"),
    "grad_missing_factor": ("grad[k * d + c] = 2.0 * (a[i] * x[i * d + c] - acc[c]);",
                            "grad[k * d + c] = (a[i] * x[i * d + c] - acc[c]);"),
    "grad_missing_weight": ("grad[k * d + c] = 2.0 * (a[i] * x[i * d + c] - acc[c]);",
                            "grad[k * d + c] = 2.0 * (x[i * d + c] - acc[c]);"),
    "cost_mass_term": ("*out = fa + gb - eps * (mass - ma * mb);", "*out = fa + gb - eps * mass;"),
    "cost_plan_weight": ("s += a[i] * b[j] * exp((f[i] + g[j] - c) / eps);",
                         "s += b[j] * exp((f[i] + g[j] - c) / eps);"),
    "init_not_zero": ("g_out[j] = g_init ? g_init[j] : 0.0;", "g_out[j] = g_init ? g_init[j] : 1.0;"),
    "g_update_stale_order": (
        "    rc = oracle_lse_update(x, n, y, m, d, b, g_out, eps, NULL, n, f_out);\n"
        "    if (rc) return rc;\n"
        "    rc = oracle_lse_update(y, m, x, n, d, a, f_out, eps, NULL, m, g_out);",
        "    rc = oracle_lse_update(y, m, x, n, d, a, f_out, eps, NULL, m, g_out);\n"
        "    if (rc) return rc;\n"
        "    rc = oracle_lse_update(x, n, y, m, d, b, g_out, eps, NULL, n, f_out);"),
    "grad_uses_f_pass_weights": ("double p = a[i] * b[j] * exp((ft[k] + g[j] - cij) / eps);",
                                 "double p = b[j] * exp((ft[k] + g[j] - cij) / eps);"),
    "symmetric_blend_swapped": ("f_out[i] = (1.0 - alpha) * f_out[i] + alpha * fn[i];",
                                "f_out[i] = alpha * f_out[i] + (1.0 - alpha) * fn[i];"),
    "symmetric_g_from_new_f": (
        "if (!rc) rc = oracle_lse_update(y, m, x, n, d, a, f_out, eps, NULL, m, gn);",
        "if (!rc) rc = oracle_lse_update(y, m, x, n, d, a, fn, eps, NULL, m, gn);"),
    "potential_reference_not_moved": ("fp[i] = f_out[i];", ";"),
    "check_cadence_off_by_one": ("it % stop_check_every != 0", "(it + 1) % stop_check_every != 0"),
    "no_check_at_the_cap": ("(it % stop_check_every != 0 && it != total)",
                            "(it % stop_check_every != 0)"),
}


def _pin_calls():
    """Every pin test, with the first parameter set of each parametrised one."""
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        kwargs = {}
        for mk in marks:
            if mk.name == "parametrize":
                argnames, values = mk.args[0], mk.args[1]
                names = [s.strip() for s in argnames.split(",")]
                first = values[0] if len(names) > 1 else (values[0],)
                kwargs.update(dict(zip(names, first)))
        calls.append((name, fn, kwargs))
    return calls


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_mutant(mutant, tmp_path, monkeypatch):
    before, after = MUTANTS[mutant]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation site for {mutant} not unique"
    mpath = tmp_path / "mutant.c"
    mpath.write_text(src.replace(before, after))
    lib_path = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o",
                    str(lib_path), str(mpath), "-lm"], check=True)
    real = oracle._load()
    lib = ctypes.CDLL(str(lib_path))
    for fname in ("oracle_lse_update", "oracle_potentials", "oracle_plan_row_sums", "oracle_cost",
                  "oracle_grad_x", "oracle_solve", "oracle_set_threads", "oracle_threads"):
        getattr(lib, fname).argtypes = getattr(real, fname).argtypes
        getattr(lib, fname).restype = getattr(real, fname).restype
    monkeypatch.setattr(oracle, "_lib", lib)
    caught = []
    with np.errstate(all="ignore"):
        for name, fn, kwargs in _pin_calls():
            try:
                fn(**kwargs)
            except Exception:  # noqa: BLE001 - any failure of a pin counts as a catch
                caught.append(name)
    assert caught, f"no pin caught mutant {mutant}"


# Mutants of the numpy transport products and Hessian-vector product (oracle/transport.py),
# loaded from an edited copy and swapped into the oracle package for the pin run.
PY_SRC = os.path.join(os.path.dirname(oracle.__file__), "transport.py")
PY_MUTANTS = {
    "hvp_dropped_direct_term": ("return 2.0 * a[:, None] * v + (2.0 / eps)",
                                "return (2.0 / eps)"),
    "hvp_flipped_cost_change": ("w = P * (df[:, None] + dg[None, :] - dC)",
                                "w = P * (df[:, None] + dg[None, :] + dC)"),
    "hvp_column_rhs_from_rows": ("s = (P * dC).sum(axis=0)", "s = (P * dC).sum(axis=0) * 0.0"),
    "hvp_plan_of_given_g_only": ("ft = f_update(x, y, b, eps, g)", "ft = np.zeros(len(x))"),
    "plan_missing_row_weight": (
        "return _d(a)[:, None] * _d(b)[None, :] * np.exp(",
        "return _d(b)[None, :] * np.exp("),
}


@pytest.mark.parametrize("mutant", sorted(PY_MUTANTS))
def test_pins_catch_python_mutant(mutant, tmp_path, monkeypatch):
    import importlib.util
    before, after = PY_MUTANTS[mutant]
    src = open(PY_SRC).read()
    assert src.count(before) == 1, f"mutation site for {mutant} not unique"
    mpath = tmp_path / "transport_mutant.py"
    mpath.write_text(src.replace(before, after))
    spec = importlib.util.spec_from_file_location("transport_mutant", mpath)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    for fname in ("hvp", "plan", "transport_apply", "transport_apply_t"):
        monkeypatch.setattr(oracle, fname, getattr(mod, fname))
    caught = []
    with np.errstate(all="ignore"):
        for name, fn, kwargs in _pin_calls():
            try:
                fn(**kwargs)
            except Exception:  # noqa: BLE001 - any failure of a pin counts as a catch
                caught.append(name)
    assert caught, f"no pin caught mutant {mutant}"
