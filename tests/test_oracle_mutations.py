"""Planted mistakes in the oracle are caught by its pins.

Each case edits one line of the oracle's source text, loads the edited copy as
a separate module (CPU only, nothing on disk changes), points the pin tests at
it and checks that at least one of the named pins fails.
"""
import importlib.util
import os
import types

import pytest

import tests.test_oracle_pins as P
from oracle import rt_oracle

SRC = open(rt_oracle.__file__).read()

MUTANTS = {
    "softmax scale 1/d_h instead of 1/sqrt(d_h)": (
        "    scale = 1.0 / np.sqrt(dh)\n    z = np.empty_like(x)",
        "    scale = 1.0 / dh\n    z = np.empty_like(x)",
        ["test_N2_closed_form_persistent_key_from_output"]),
    "persistent pair taken from the input": (
        'src = zt if kv_source == "output" else x[:, t]', "src = x[:, t]",
        ["test_N2_closed_form_persistent_key_from_output"]),
    "dropped attention residual": (
        'u = x[:, t] + a.reshape(B, d) @ W["W_o"].T', 'u = a.reshape(B, d) @ W["W_o"].T',
        ["test_N1_closed_form_single_token_layer"]),
    "transposed W_o": (
        'u = x[:, t] + a.reshape(B, d) @ W["W_o"].T', 'u = x[:, t] + a.reshape(B, d) @ W["W_o"]',
        ["test_N1_closed_form_single_token_layer"]),
    "tanh-approximate GELU": (
        "return 0.5 * y * (1.0 + erf(y / np.sqrt(2.0)))",
        "return 0.5 * y * (1.0 + np.tanh(0.7978845608028654 * (y + 0.044715 * y ** 3)))",
        ["test_gelu_matches_normal_cdf_values"]),
    "eps outside the mean": (
        "np.mean(v * v, axis=-1, keepdims=True) + EPS", "np.sum(v * v, axis=-1, keepdims=True) + EPS",
        ["test_rms_definition"]),
    "key block one short": (
        "keys = list(range(t - lb + 1, t + 1))", "keys = list(range(t - lb + 2, t + 1))",
        ["test_schedule_covers_every_causal_pair_exactly_once"]),
    "query block one short": (
        "queries = list(range(t + 1, min(t + lb, N) + 1))", "queries = list(range(t + 1, min(t + lb, N)))",
        ["test_schedule_covers_every_causal_pair_exactly_once"]),
    "decode step: persistent pair from the input": (
        "    rz = rms(z_t)\n    return z_t, rz @ W[\"W_k\"].T, rz @ W[\"W_v\"].T",
        "    rz = rms(x_t)\n    return z_t, rz @ W[\"W_k\"].T, rz @ W[\"W_v\"].T",
        ["test_decode_step_N1_closed_form", "test_decode_from_empty_cache_reproduces_the_layer"]),
    "decode step: temporary key used as its value": (
        "    vals = np.concatenate([V_prev, v_tmp[:, :, None]], axis=2)",
        "    vals = np.concatenate([V_prev, k_tmp[:, :, None]], axis=2)",
        ["test_decode_step_N1_closed_form", "test_decode_from_empty_cache_reproduces_the_layer"]),
    "paper parameterisation: softmax scale kept": (
        '        s = np.einsum("bhe,bhie->bhi", q, keys)\n        w = np.exp(s - s.max',
        '        s = np.einsum("bhe,bhie->bhi", q, keys) / np.sqrt(dh)\n        w = np.exp(s - s.max',
        ["test_pages_parameterisation_N1_N2_closed_forms", "test_pages_parameterisation_standard_layer_reduction"]),
    "paper parameterisation: query norm over the whole width": (
        '        q = rms_unit(_heads(r @ W["W_q"].T, H))',
        '        q = _heads(rms_unit(r @ W["W_q"].T), H)',
        ["test_pages_parameterisation_N1_N2_closed_forms", "test_pages_parameterisation_standard_layer_reduction"]),
    "paper parameterisation: attention residual not scaled": (
        '        u = x[:, t] + (a.reshape(B, d) @ W["W_o"].T) * inv_sqrt_L',
        '        u = x[:, t] + (a.reshape(B, d) @ W["W_o"].T)',
        ["test_pages_parameterisation_N1_N2_closed_forms"]),
    "wrong rescale sign in the fold": (
        "alpha = np.where(np.isneginf(m), 0.0, np.exp(m - m_new))",
        "alpha = np.where(np.isneginf(m), 0.0, np.exp(m_new - m))",
        ["test_blocked_equals_naive", "test_block_fold_equals_direct_softmax_and_is_associative"]),
}


def _load_mutant(old, new):
    assert SRC.count(old) >= 1, old
    mod = types.ModuleType("rt_oracle_mutant")
    mod.__file__ = rt_oracle.__file__
    exec(compile(SRC.replace(old, new, 1), "rt_oracle_mutant", "exec"), mod.__dict__)
    return mod


def _run_pin(name):
    fn = getattr(P, name)
    if name == "test_schedule_covers_every_causal_pair_exactly_once":
        for N in (8, 13, 64):
            fn(N)
    elif name == "test_blocked_equals_naive":
        for N in (3, 8, 64):
            fn(N)
    else:
        fn()


@pytest.mark.parametrize("label", list(MUTANTS))
def test_pins_catch_planted_mistake(label, monkeypatch):
    old, new, pins = MUTANTS[label]
    monkeypatch.setattr(P, "O", _load_mutant(old, new))
    caught = False
    for name in pins:
        try:
            _run_pin(name)
        except AssertionError:
            caught = True
    assert caught, f"no pin caught: {label}"


def test_unmutated_copy_passes_the_same_pins(monkeypatch):
    monkeypatch.setattr(P, "O", _load_mutant("EPS = 1e-6", "EPS = 1e-6"))
    for _, _, pins in MUTANTS.values():
        for name in pins:
            _run_pin(name)
