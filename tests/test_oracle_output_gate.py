"""Pins of the oracle's output normalisation and gate (RMSNorm per head and a
sigmoid output gate, the "Kimi Linear" summary's section on the model
configuration), checked against hand-worked values and identities of the
definition rather than against the formula retyped."""
import numpy as np
import pytest

import oracle

BIG = 40.0  # sigmoid(40) = 1 - 4e-18: the gate fully open in fp64


def test_hand_worked_two_channels():
    out = oracle.output_gate(np.array([[3.0, 4.0]]), np.full((1, 2), BIG), np.ones(2), 0.0)
    # rms = sqrt((9 + 16) / 2) = sqrt(12.5)
    assert np.allclose(out, [[3.0 / 12.5 ** 0.5, 4.0 / 12.5 ** 0.5]], rtol=1e-15, atol=0)
    assert np.allclose(out, [[0.8485281374238571, 1.1313708498984762]], rtol=1e-15, atol=0)


def test_closed_gate_halves_and_sigmoid_symmetry():
    rng = np.random.default_rng(1)
    o = rng.standard_normal((5, 16))
    w = rng.uniform(0.5, 2.0, 16)
    g = rng.standard_normal((5, 16))
    open_ = oracle.output_gate(o, np.full_like(o, BIG), w, 1e-6)
    half = oracle.output_gate(o, np.zeros_like(o), w, 1e-6)
    assert np.allclose(half, 0.5 * open_, rtol=1e-15, atol=0)
    # sigmoid(x) + sigmoid(-x) = 1
    both = oracle.output_gate(o, g, w, 1e-6) + oracle.output_gate(o, -g, w, 1e-6)
    assert np.allclose(both, open_, rtol=1e-13, atol=1e-15)


def test_scale_invariance_and_unit_rms_per_row():
    rng = np.random.default_rng(2)
    o = rng.standard_normal((7, 128)) * rng.uniform(0.01, 100.0, (7, 1))
    g = np.full_like(o, BIG)
    out = oracle.output_gate(o, g, np.ones(128), 0.0)
    assert np.allclose(np.mean(out ** 2, axis=1), 1.0, rtol=1e-13)
    assert np.allclose(oracle.output_gate(3.7 * o, g, np.ones(128), 0.0), out, rtol=1e-13, atol=1e-15)


def test_rows_are_independent_and_weight_is_per_channel():
    rng = np.random.default_rng(3)
    o = rng.standard_normal((6, 32))
    g = rng.standard_normal((6, 32))
    w = rng.uniform(0.5, 2.0, 32)
    out = oracle.output_gate(o, g, w, 1e-5)
    perm = rng.permutation(6)
    assert np.array_equal(oracle.output_gate(o[perm], g[perm], w, 1e-5), out[perm])
    w2 = w.copy()
    w2[5] *= 2.0
    out2 = oracle.output_gate(o, g, w2, 1e-5)
    assert np.allclose(out2[:, 5], 2.0 * out[:, 5], rtol=1e-15)
    assert np.array_equal(np.delete(out2, 5, axis=1), np.delete(out, 5, axis=1))


def test_epsilon_inside_the_root():
    o = np.full((1, 8), 1e-3)
    out = oracle.output_gate(o, np.full_like(o, BIG), np.ones(8), 1.0)
    assert np.allclose(out, 1e-3 / np.sqrt(1e-6 + 1.0), rtol=1e-15)
    zero = oracle.output_gate(np.zeros((2, 8)), np.zeros((2, 8)), np.ones(8), 1e-5)
    assert np.all(zero == 0.0)


def test_bad_arguments_are_refused():
    with pytest.raises(ValueError):
        oracle.output_gate(np.ones((2, 4)), np.ones((2, 3)), np.ones(4), 0.0)
    with pytest.raises(ValueError):
        oracle.output_gate(np.ones((2, 4)), np.ones((2, 4)), np.ones(4), -1.0)
