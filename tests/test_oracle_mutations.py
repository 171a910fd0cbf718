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
import tests.test_oracle_bwd_pins as bwd_pins
import tests.test_oracle_kda_pins as kda_pins
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")

MUTATIONS = {
    "residual_without_alpha": ("const double u = beta * (vt[i] - alpha * x[i]);",
                               "const double u = beta * (vt[i] - x[i]);"),
    "write_without_beta": ("const double u = beta * (", "const double u = ("),
    "state_not_transposed": ("S[(size_t)i * dk + j] = st[(size_t)j * dv + i];",
                             "S[(size_t)i * dk + j] = st[(size_t)i * dk + j];"),
    "gate_ignored": ("const double alpha = exp(J->g[row]);", "const double alpha = 1.0;"),
    "update_sign": ("alpha * S[(size_t)i * dk + j] + u * kt[j]",
                    "alpha * S[(size_t)i * dk + j] - u * kt[j]"),
    "gate_on_write_only": ("S[(size_t)i * dk + j] = alpha * S[(size_t)i * dk + j] + u * kt[j];",
                           "S[(size_t)i * dk + j] = S[(size_t)i * dk + j] + u * kt[j];"),
}

# Mistakes in the channel-wise-gate loop, caught by its own pins.
KDA_MUTATIONS = {
    "kda_gate_ignored": ("for (int j = 0; j < dk; ++j) a[j] = exp(gt[j]);",
                         "for (int j = 0; j < dk; ++j) a[j] = 1.0;"),
    "kda_residual_from_undecayed_state": (
        "acc += S[(size_t)i * dk + j] * a[j] * kt[j];",
        "acc += S[(size_t)i * dk + j] * kt[j];"),
    "kda_decay_after_write": (
        "S[(size_t)i * dk + j] = a[j] * S[(size_t)i * dk + j] + ui * kt[j];",
        "S[(size_t)i * dk + j] = a[j] * (S[(size_t)i * dk + j] + ui * kt[j]);"),
    "kda_decay_on_value_axis": (
        "S[(size_t)i * dk + j] = a[j] * S[(size_t)i * dk + j] + ui * kt[j];",
        "S[(size_t)i * dk + j] = a[i % dk] * S[(size_t)i * dk + j] + ui * kt[j];"),
    "kda_gate_of_previous_token": (
        "const double *gt = J->g + row * dk;",
        "const double *gt = J->g + (row >= (size_t)H ? row - H : row) * dk;"),
}

KDA_PIN_CASES = [
    kda_pins.test_kda_hand_worked_two_tokens,
    kda_pins.test_kda_equal_channels_is_scalar_gate,
    kda_pins.test_kda_beta_zero_is_channel_decay,
    lambda: kda_pins.test_kda_unit_key_beta_one_overwrites(3),
    lambda: kda_pins.test_kda_dense_chunked_matches_token_loop(4, 7),
    kda_pins.test_kda_cycling_unit_keys_closed_form,
]

# Mistakes in the gradient loop, caught by the gradient pins.
BWD_MUTATIONS = {
    "bwd_dk_without_state_term": (
        "acc += G[(size_t)i * dk + j] * u[i] - alpha * beta * Sp[(size_t)i * dk + j] * Gk[i];",
        "acc += G[(size_t)i * dk + j] * u[i];"),
    "bwd_carry_without_beta": (
        "G[(size_t)i * dk + j] = alpha * (G[(size_t)i * dk + j] - beta * Gk[i] * kt[j]);",
        "G[(size_t)i * dk + j] = alpha * (G[(size_t)i * dk + j] - Gk[i] * kt[j]);"),
    "bwd_dg_without_alpha": ("J->dg[row] = alpha * (gs - beta * gx);",
                             "J->dg[row] = gs - beta * gx;"),
    "bwd_dq_from_previous_state": (
        "acc += (alpha * Sp[(size_t)i * dk + j] + u[i] * kt[j]) * dot[i];",
        "acc += Sp[(size_t)i * dk + j] * dot[i];"),
    "bwd_output_grad_not_added": ("for (int j = 0; j < dk; ++j) G[(size_t)i * dk + j] += dot[i] * qt[j];",
                                  "for (int j = 0; j < dk; ++j) G[(size_t)i * dk + j] += 0.0 * qt[j];"),
}

BWD_PIN_CASES = [
    lambda: bwd_pins.test_bwd_matches_central_differences("plain"),
    bwd_pins.test_bwd_homogeneity_identities,
    bwd_pins.test_bwd_beta_zero_closed_form,
    bwd_pins.test_bwd_is_causal,
]

PIN_CASES = [
    pins.test_hand_worked_two_tokens,
    pins.test_beta_zero_is_pure_decay,
    pins.test_alpha_one_first_token_closed_form,
    pins.test_unit_key_beta_one_overwrites,
    pins.test_orthogonal_direction_only_decays,
    lambda: pins.test_orthogonal_keys_closed_form(True),
    lambda: pins.test_dense_chunked_matches_token_loop(4, 7),
]


ALL = {**{n: (m, PIN_CASES) for n, m in MUTATIONS.items()},
       **{n: (m, KDA_PIN_CASES) for n, m in KDA_MUTATIONS.items()},
       **{n: (m, BWD_PIN_CASES) for n, m in BWD_MUTATIONS.items()}}


@pytest.mark.parametrize("name", sorted(ALL))
def test_planted_mistake_is_caught(name, tmp_path, monkeypatch):
    (before, after), cases = ALL[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "mut.c"
    mutated.write_text(src.replace(before, after))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-shared", "-fPIC", "-pthread",
                           str(mutated), "-o", str(so), "-lm"])
    real = oracle._load()
    lib = ctypes.CDLL(str(so))
    for fn in ("gdn_oracle_chunk_fwd", "gdn_oracle_decode_step", "gdn_oracle_kda_chunk_fwd",
               "gdn_oracle_kda_decode_step", "gdn_oracle_chunk_bwd"):
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
        getattr(lib, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", lib)
    failures = 0
    for case in cases:
        try:
            case()
        except AssertionError:
            failures += 1
    assert failures >= 1, f"no pin noticed the planted mistake {name}"
