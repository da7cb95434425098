"""Every plausible slip in the oracle must fail at least one pin.

Each mutant is a copy of ``oracle/kda_oracle.c`` with one deliberate mistake,
compiled into a temporary library on the CPU.  The pin checks from
``test_oracle_pins`` run against it with the oracle's library handle swapped;
at least one must fail.  This shows the pins are not vacuous.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")

DECAY = "for (int64_t j = 0; j < d; ++j) row[j] *= a;"
UPDATE = "row[j] += bk * (v[j] - u[j]);"
READ = "o[j] += row[j] * qi;"


def _swap_blocks(src, first_marker, second_marker, end_marker):
    a = src.index(first_marker)
    b = src.index(second_marker)
    c = src.index(end_marker)
    return src[:a] + src[b:c] + src[a:b] + src[c:]


MUTANTS = {
    "decay_on_value_axis": lambda s: s.replace(DECAY, "for (int64_t j = 0; j < d; ++j) row[j] *= exp(g[j]);"),
    "decay_sign": lambda s: s.replace("double a = exp(g[i]);", "double a = exp(-g[i]);"),
    "no_erase": lambda s: s.replace(UPDATE, "row[j] += bk * v[j];"),
    "erase_sign": lambda s: s.replace(UPDATE, "row[j] += bk * (v[j] + u[j]);"),
    "no_beta": lambda s: s.replace("double bk = beta * k[i];", "double bk = k[i];"),
    "readout_S_not_ST": lambda s: s.replace(READ, "o[i] += row[j] * q[j];"),
    "readout_before_update": lambda s: _swap_blocks(s, "    /* S = S' + beta", "    /* o = scale",
                                                    "    for (int64_t j = 0; j < d; ++j) o[j] *= scale;"),
    "erase_before_decay": lambda s: _swap_blocks(s, "    /* S' = Diag(alpha) S", "    /* u = S'^T k",
                                                 "    /* S = S' + beta"),
    "norm_without_sqrt": lambda s: s.replace("1.0 / sqrt(ss + eps)", "1.0 / (ss + eps)"),
    "no_scale": lambda s: s.replace("for (int64_t j = 0; j < d; ++j) o[j] *= scale;", ""),
    "initial_state_ignored": lambda s: s.replace("if (initial_state)\n", "if (0)\n"),
}

PIN_CHECKS = [
    pins.test_golden_worked_example_exact,
    pins.test_golden_worked_example_with_l2norm,
    pins.test_I1_beta0_alpha1_leaves_state_unchanged,
    pins.test_I2_delta_overwrite_reads_back_v,
    pins.test_I4_beta0_closed_form_decay,
    lambda: pins.test_I5_bruteforce_matrix_products(True),
    pins.test_I9_order_of_decay_and_erase,
]


def _build_mutant(tmp_path, name, mutate):
    src = open(SRC).read()
    mutated = mutate(src)
    assert mutated != src, f"mutation {name} did not apply"
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(mutated)
    subprocess.run(["gcc", "-O1", "-fopenmp", "-shared", "-fPIC", "-std=c99", str(c), "-o", str(so),
                    "-lm"], check=True)
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path, monkeypatch):
    so = _build_mutant(tmp_path, name, MUTANTS[name])
    real = oracle._load()
    lib = ctypes.CDLL(so)
    for fn in ("kda_oracle_forward", "kda_oracle_decode", "kda_oracle_max_threads"):
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
        getattr(lib, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", lib)
    failures = 0
    for check in PIN_CHECKS:
        try:
            check()
        except AssertionError:
            failures += 1
    assert failures > 0, f"mutant {name} passed every pin"
