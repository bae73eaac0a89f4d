"""Plant plausible mistakes in copies of the oracle's C source and check that
the pins catch every one (CPU only).

Each mutant is compiled into a temporary library and swapped in for the real
oracle; the pin functions from ``test_oracle_pins`` then run against it.  A
mutant that passes every pin would mean the pins leave that part of the oracle
unchecked.
"""
import ctypes
import os

import numpy as np
import pytest

import oracle.build as obuild
import oracle.kda_oracle as ko
from tests import test_oracle_pins as pins

MUTANTS = {
    "no_decay": ("S[i * dv + j] *= a;", "S[i * dv + j] *= 1.0;"),
    "decay_sign": ("exp(gt[i])", "exp(-gt[i])"),
    "decay_on_columns": ("S[i * dv + j] *= a;", "S[i * dv + j] *= exp(gt[j % dk]);"),
    "erase_sign": ("- bt * kt[i] * u[j]", "+ bt * kt[i] * u[j]"),
    "erase_dropped": ("- bt * kt[i] * u[j]", ""),
    "write_dropped": ("+ bt * kt[i] * vt[j]", ""),
    "erase_reads_query": ("u[j] += kt[i] * S[i * dv + j];", "u[j] += qt[i] * S[i * dv + j];"),
    "read_uses_key": ("ot[j] += qt[i] * S[i * dv + j];", "ot[j] += kt[i] * S[i * dv + j];"),
    "beta_squared": ("const double bt = beta[t * H + h];",
                     "const double bt = beta[t * H + h] * beta[t * H + h];"),
    "beta_of_previous_token": ("const double bt = beta[t * H + h];",
                               "const double bt = beta[(t > t0 ? t - 1 : t) * H + h];"),
    "read_before_update": ("        /* o_t = S_t^T q_t. */",
                           "        /* o_t = S_t^T q_t. */ continue;"),
    "initial_state_ignored": ("if (src != S) memmove(S, src, sizeof(double) * (size_t)(dk * dv));",
                              "memset(S, 0, sizeof(double) * (size_t)(dk * dv));"),
}

PIN_FUNCS = [
    lambda: pins.test_brute_force_operator_products(12, 4, 4, 2),
    lambda: pins.test_brute_force_operator_products(9, 2, 5, 3),
    pins.test_exact_rational_arithmetic,
    pins.test_beta_zero_is_pure_decay,
    pins.test_unit_write_retrieves_last_value,
    pins.test_orthonormal_keys_are_an_associative_memory,
    pins.test_scalar_key_dimension_closed_form,
    lambda: pins.test_chunked_evaluation_equals_recurrence(16),
]


def _load(path):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lp = ctypes.POINTER(ctypes.c_int64)
    lib.kda_oracle_fwd.argtypes = [dp, dp, dp, dp, dp, dp, lp, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_int64, ctypes.c_int64, ctypes.c_int, dp, dp]
    lib.kda_oracle_fwd.restype = ctypes.c_int
    return lib


def test_unmutated_oracle_passes_every_pin():
    for f in PIN_FUNCS:
        f()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path, monkeypatch):
    before, after = MUTANTS[name]
    src = open(obuild.SRC).read()
    assert before in src, f"mutation site for {name} not found"
    mut_src = tmp_path / f"{name}.c"
    mut_src.write_text(src.replace(before, after, 1))
    lib_path = str(tmp_path / f"lib{name}.so")
    obuild.build(force=True, src=str(mut_src), out=lib_path)
    monkeypatch.setattr(ko, "_LIB", _load(lib_path))
    caught = 0
    for f in PIN_FUNCS:
        try:
            with np.errstate(all="ignore"):
                f()
        except AssertionError:
            caught += 1
    assert caught > 0, f"mutant {name} passed every pin"
    assert os.path.exists(lib_path)
