"""Plant plausible mistakes in a copy of the oracle (CPU only) and check that
the pins in test_oracle_pins.py catch every one of them."""
import importlib.util
import os
import types

import numpy as np
import pytest

import oracle as O
import workloads as W
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "zo_oracle.py")

MUTATIONS = {
    "swap_i_f_gates": ("i = _sigmoid(G[:, 0:H])\n            f = _sigmoid(G[:, H:2 * H])",
                       "f = _sigmoid(G[:, 0:H])\n            i = _sigmoid(G[:, H:2 * H])"),
    "drop_cell_bias": (' @ W.T + P[f"b{l + 1}"]', " @ W.T"),
    "no_recurrent_feed": ("            x = h[l]\n", "            pass\n"),
    "tanh_for_sigmoid_o": ("o = _sigmoid(G[:, 3 * H:4 * H])", "o = np.tanh(G[:, 3 * H:4 * H])"),
    "missing_factor_two": ("return h * (lp - lm) / (2.0 * e * n_pert)", "return h * (lp - lm) / (e * n_pert)"),
    "wrong_update_sign": ("return th - np.asarray(coeffs", "return th + np.asarray(coeffs"),
    "philox_no_key_xor": ("hi1 ^ c1 ^ np.uint64(k0)", "hi1 ^ c1"),
    "philox_no_key_bump": ("k0 = (k0 + PHILOX_W0) & 0xFFFFFFFF", "k0 = k0"),
    "philox_swapped_multipliers": ("p0 = c0 * np.uint64(PHILOX_M0)", "p0 = c0 * np.uint64(PHILOX_M1)"),
    "lse_without_max": ("lse = m[:, 0] + np.log", "lse = np.log"),
    "perturb_ignores_sign": ("+ sign * e * p", "+ e * p"),
    "gram_cosine_no_sqrt": ("den = math.sqrt(max(a @ gram @ a, 0.0) * max(b @ gram @ b, 0.0))",
                            "den = max(a @ gram @ a, 0.0) * max(b @ gram @ b, 0.0)"),
    "gram_cosine_ignores_gram": ("num = a @ gram @ b", "num = a @ b"),
    "gram_counts_padding": ("        cnt = r * c\n        S = np.stack",
                            "        cnt = -(-(r * c) // 128) * 128\n        S = np.stack"),
    "gram_ignores_probe_list": ("S = np.stack([probe_signs(step_seed, i, off, cnt).astype(np.int64) for i in probes])",
                                "S = np.stack([probe_signs(step_seed, i, off, cnt).astype(np.int64) for i in range(n)])"),
}


def mutant(name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, name
    mod = types.ModuleType("zo_oracle_mutant")
    exec(compile(src.replace(old, new), SRC, "exec"), mod.__dict__)
    return mod


PIN_FUNCS = [
    pins.test_philox_known_answers,
    lambda: pins.test_forward_matches_torch_lstm(7, 5, 6, 3, 4, 9, 0.3),
    pins.test_quadratic_all_sign_vectors_give_exact_gradient,
    pins.test_central_difference_matches_directional_derivative,
    pins.test_antisymmetry_negated_probe_negates_coefficient,
    pins.test_probe_gram_matches_explicit_products,
    pins.test_gram_cosine_hand_values,
    pins.test_gram_cosine_equals_cosine_of_explicit_estimates,
]


def _some_pin_fails(mod, monkeypatch):
    monkeypatch.setattr(pins, "O", mod)
    for f in PIN_FUNCS:
        try:
            f()
        except Exception:
            return True
    return False


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    mod = mutant(name)
    with np.errstate(all="ignore"):
        assert _some_pin_fails(mod, monkeypatch), f"no pin caught mutation {name}"


def test_unmutated_copy_passes_the_same_pins(monkeypatch):
    src = open(SRC).read()
    mod = types.ModuleType("zo_oracle_copy")
    exec(compile(src, SRC, "exec"), mod.__dict__)
    assert not _some_pin_fails(mod, monkeypatch)
