"""Planted mistakes in the oracle must each fail at least one pin (CPU only).

Each mutant is a textual edit of a copy of oracle/kda_oracle.c, compiled into
a temporary library; the oracle source itself is never changed.
"""
import functools
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")

MUTANTS = {
    "beta_dropped": [("u[j] = bt * (vt[j] - u[j]);", "u[j] = (vt[j] - u[j]);")],
    "error_sign": [("u[j] = bt * (vt[j] - u[j]);", "u[j] = bt * (vt[j] + u[j]);")],
    "decay_after_delta": [
        ("for (int j = 0; j < nc; ++j) row[j] *= a[i];", ""),
        ("for (int j = 0; j < nc; ++j) row[j] += ki * u[j];",
         "for (int j = 0; j < nc; ++j) row[j] = (row[j] + ki * u[j]) * a[i];"),
    ],
    "output_before_write": [("ot[j] += qi * row[j];", "ot[j] += qi * (row[j] - kt[i] * u[j]);")],
    "recall_with_q": [("u[j] += ki * row[j];", "u[j] += qt[i] * row[j];")],
    "gate_channel_shift": [("a[i] = exp(lat[i]);", "a[i] = exp(lat[(i + 1) % dk]);")],
    "gate_ignored": [("a[i] = exp(lat[i]);", "a[i] = 1.0;")],
    "s0_ignored": [("J->S0 ? J->S0[soff + (size_t)i * dv + j] : 0.0", "0.0")],
    "value_column_offset": [("* dv + j0;\n        const double bt", "* dv;\n        const double bt")],
    "beta_head_index": [("J->beta[(size_t)t * H + h]", "J->beta[(size_t)t * H]")],
    "state_not_written": [("J->S_T[soff + (size_t)i * dv + j] = S[(size_t)i * nc + (j - j0)];",
                           "J->S_T[soff + (size_t)i * dv + j] = J->S0 ? J->S0[soff + (size_t)i * dv + j] : 0.0;")],
}


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return tmp_path_factory.mktemp("oracle_mutants")


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, mutant_dir):
    src = open(SRC, encoding="utf-8").read()
    for old, new in MUTANTS[name]:
        assert old in src, f"mutation anchor for {name} not found in the oracle source"
        src = src.replace(old, new)
    c_path = os.path.join(mutant_dir, f"{name}.c")
    with open(c_path, "w", encoding="utf-8") as f:
        f.write(src)
    so = oracle.compile_oracle(c_path, os.path.join(mutant_dir, f"{name}.so"))
    fwd = functools.partial(oracle.kda_fwd, lib_path=so)
    failed = []
    for pin in ALL_PINS:
        try:
            pin(fwd)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
