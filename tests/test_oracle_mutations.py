"""Planted mistakes in the oracle must be caught by its pins.

Each case edits a copy of the C oracle's source (on the CPU, in a temporary
directory), builds it, swaps it in for the real library and runs the pin
tests; at least one pin must fail. This shows the pins are strong enough to
notice a dropped term, a wrong sign, a transposed state or a missing gate.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")

MUTATIONS = {
    "residual_without_alpha": ("(vt[i] - alpha * x[i])", "(vt[i] - x[i])"),
    "write_without_beta": ("const double u = beta * (", "const double u = ("),
    "state_not_transposed": ("S[(size_t)i * dk + j] = st[(size_t)j * dv + i];",
                             "S[(size_t)i * dk + j] = st[(size_t)i * dk + j];"),
    "gate_ignored": ("const double alpha = exp(J->g[row]);", "const double alpha = 1.0;"),
    "update_sign": ("alpha * S[(size_t)i * dk + j] + u * kt[j]",
                    "alpha * S[(size_t)i * dk + j] - u * kt[j]"),
    "gate_on_write_only": ("S[(size_t)i * dk + j] = alpha * S[(size_t)i * dk + j] + u * kt[j];",
                           "S[(size_t)i * dk + j] = S[(size_t)i * dk + j] + u * kt[j];"),
}

PIN_CASES = [
    pins.test_hand_worked_two_tokens,
    pins.test_beta_zero_is_pure_decay,
    pins.test_alpha_one_first_token_closed_form,
    pins.test_unit_key_beta_one_overwrites,
    pins.test_orthogonal_direction_only_decays,
    lambda: pins.test_orthogonal_keys_closed_form(True),
    lambda: pins.test_dense_chunked_matches_token_loop(4, 7),
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path, monkeypatch):
    before, after = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "mut.c"
    mutated.write_text(src.replace(before, after))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-shared", "-fPIC", "-pthread",
                           str(mutated), "-o", str(so), "-lm"])
    real = oracle._load()
    lib = ctypes.CDLL(str(so))
    for fn in ("gdn_oracle_chunk_fwd", "gdn_oracle_decode_step"):
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
        getattr(lib, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", lib)
    failures = 0
    for case in PIN_CASES:
        try:
            case()
        except AssertionError:
            failures += 1
    assert failures >= 1, f"no pin noticed the planted mistake {name}"
