"""The pins are strong enough: plant one plausible mistake at a time in a copy
of the oracle source (on the CPU), rebuild it, and check that at least one pin
of tests/test_oracle_pins.py fails on it.

Every mutant keeps all memory accesses in bounds (only values, signs, index
orders inside the same buffer, or operands change).
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from oracle import Oracle
import test_oracle_pins as pins

SRC = open(oracle.SRC).read()

MUTANTS = {
    "silu_sign": ("z / (1.0 + exp(-z))", "z / (1.0 + exp(z))"),
    "silu_dropped": ("for (int r = 0; r < R; ++r) z[r] = silu(z[r]);", ""),
    "w2_transposed": ("acc += z[r] * W2[(long)r * HW + c];", "acc += z[r] * W2[(long)c * R + r];"),
    "conv_taps_reversed": ("acc += wt[j] * v_at(", "acc += wt[W - 1 - j] * v_at("),
    "conv_history_reversed": ("hist[(((long)b * (W - 1) + m) * H + h)", "hist[(((long)b * (W - 1) + (W - 2 - m)) * H + h)"),
    "gdn_gate_not_on_erase": ("Si[j] = a * (Si[j] - bt * u * kh[j]) + bt * vi * kh[j];",
                              "Si[j] = a * Si[j] - bt * u * kh[j] + bt * vi * kh[j];"),
    "gdn_gate_on_write": ("Si[j] = a * (Si[j] - bt * u * kh[j]) + bt * vi * kh[j];",
                          "Si[j] = a * (Si[j] - bt * u * kh[j] + bt * vi * kh[j]);"),
    "gdn_delta_sign": ("Si[j] = a * (Si[j] - bt * u * kh[j])", "Si[j] = a * (Si[j] + bt * u * kh[j])"),
    "gdn_output_uses_key": ("for (int j = 0; j < dk; ++j) oi += Si[j] * qh[j];\n                    o[bth",
                            "for (int j = 0; j < dk; ++j) oi += Si[j] * kh[j];\n                    o[bth"),
    "gdn_gate_not_exponentiated": ("const double a = exp(g[bth]), bt = beta[bth];",
                                   "const double a = g[bth] + 1.0, bt = beta[bth];"),
    "l2norm_squared": ("const double inv = 1.0 / sqrt(ss + eps);", "const double inv = 1.0 / (ss + eps);"),
    "l2norm_skipped": ("const double inv = 1.0 / sqrt(ss + eps);", "const double inv = 1.0;"),
    "l2norm_eps_outside_sqrt": ("const double inv = 1.0 / sqrt(ss + eps);", "const double inv = 1.0 / (sqrt(ss) + eps);"),
    "decode_gate_on_write": ("const double c = bt * v[bh * dv + i] - a * bt * u;",
                             "const double c = a * bt * v[bh * dv + i] - a * bt * u;"),
    "chunked_decay_sign": ("a = br * exp(G[r] - G[i]) * kk;", "a = br * exp(G[i] - G[r]) * kk;"),
    "chunked_state_no_decay": ("double s = gL * S[(long)c * dk + j];", "double s = S[(long)c * dk + j];"),
}

# pins run against each mutant (function, kwargs)
PINS = [
    (pins.test_generator_hand_worked, {}),
    (pins.test_generator_silu_closed_form_and_selection, {}),
    (pins.test_generator_linear_in_W2_and_nonlinear_in_x, {}),
    (pins.test_conv_hand_worked, {}),
    (pins.test_conv_unit_tap_is_shift, {"tap": 1}),
    (pins.test_conv_history_continuation, {"split": 2}),
    (pins.test_gdn_hand_worked, {}),
    (pins.test_gdn_sequential_equals_transition_products, {"seed": 1, "s0": True}),
    (pins.test_gdn_alpha1_beta0_leaves_state, {}),
    (pins.test_gdn_orthonormal_keys_store_values_exactly, {}),
    (pins.test_gdn_beta0_decays_state, {}),
    (pins.test_gdn_delta_rule_overwrites, {}),
    (pins.test_gdn_chunked_equals_sequential, {"T": 65, "C": 64, "long_memory": False}),
    (pins.test_gdn_decode_steps_equal_sequential, {}),
    (pins.test_gdn_l2_normalises_q_and_k, {}),
    (pins.test_gdn_l2_norm_eps_on_zero_and_tiny_vectors, {}),
    (pins.test_mixer_prefill_then_decode_continues, {}),
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_planted_mistake_fails_a_pin(name, tmp_path):
    old, new = MUTANTS[name]
    assert SRC.count(old) >= 1, f"mutation site for {name} not found"
    src = tmp_path / "mutant.c"
    src.write_text(SRC.replace(old, new, 1))
    lib = tmp_path / "libmutant.so"
    oracle.build(str(src), str(lib), force=True)
    orc = Oracle(str(lib))
    caught = []
    with np.errstate(all="ignore"):
        for fn, kw in PINS:
            try:
                fn(orc, **kw)
            except AssertionError:
                caught.append(fn.__name__)
    assert caught, f"mutant {name} passed every pin"
