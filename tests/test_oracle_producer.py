"""Pins of the oracle's producer steps: the L2 normalisation of q and k and
the channel-wise decay gate ("Kimi Linear" summary, section "Configuração do
modelo Kimi Linear"), checked against hand-worked values, closed forms
computed another way, and identities of the definitions."""
import numpy as np
import pytest

import oracle
from gated_delta_rule_110_b200 import inputs as gen


def test_l2norm_hand_worked_and_unit_rows():
    assert np.allclose(oracle.l2norm(np.array([[3.0, 4.0]]), 0.0), [[0.6, 0.8]], rtol=1e-15, atol=0)
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 3, 16)) * rng.uniform(0.01, 50.0, (5, 3, 1))
    y = oracle.l2norm(x, 0.0)
    assert np.allclose(np.linalg.norm(y, axis=-1), 1.0, rtol=1e-14)
    # same direction: y . x = |x|
    assert np.allclose(np.sum(y * x, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    # scale invariance per row, and rows independent of each other
    s = rng.uniform(0.1, 10.0, (5, 3, 1))
    assert np.allclose(oracle.l2norm(s * x, 0.0), y, rtol=1e-13, atol=1e-15)


def test_l2norm_epsilon_inside_the_root():
    x = np.full((2, 4), 0.5)  # |x|^2 = 1
    assert np.allclose(oracle.l2norm(x, 3.0), x / 2.0, rtol=1e-15)
    assert np.all(oracle.l2norm(np.zeros((3, 8)), 1e-6) == 0.0)


def test_decay_gate_hand_worked():
    la = oracle.decay_gate(np.zeros((1, 1, 2)), np.zeros(1), np.zeros((1, 2)))
    assert np.allclose(la, -np.log(2.0), rtol=1e-15)
    # A_log = log 3 triples the rate; bias 1 with f = -1 is softplus(0) again
    la = oracle.decay_gate(np.full((1, 1, 2), -1.0), np.array([np.log(3.0)]), np.ones((1, 2)))
    assert np.allclose(la, -3.0 * np.log(2.0), rtol=1e-14)


def test_decay_gate_closed_form_as_a_power():
    # alpha = exp(-e^A softplus(x)) = (1 + e^x)^(-e^A)
    rng = np.random.default_rng(1)
    H, dk = 3, 8
    f = rng.standard_normal((6, H, dk)) * 3.0
    A = rng.uniform(-1.0, 2.0, H)
    b = rng.uniform(-5.0, 1.0, (H, dk))
    alpha = np.exp(oracle.decay_gate(f, A, b))
    x = f + b[None]
    ref = np.power(1.0 + np.exp(x), -np.exp(A)[None, :, None])
    assert np.allclose(alpha, ref, rtol=1e-12, atol=0)


def test_decay_gate_limits_sign_and_indexing():
    H, dk = 2, 4
    A = np.array([0.0, np.log(2.0)])
    b = np.zeros((H, dk))
    # large argument: -e^A (x + e^-x); very negative: -e^A e^x
    big = oracle.decay_gate(np.full((1, H, dk), 40.0), A, b)
    assert np.allclose(big, -np.exp(A)[None, :, None] * 40.0, rtol=1e-15)
    small = oracle.decay_gate(np.full((1, H, dk), -40.0), A, b)
    assert np.allclose(small, -np.exp(A)[None, :, None] * np.exp(-40.0), rtol=1e-12)
    rng = np.random.default_rng(2)
    f = np.sort(rng.standard_normal(50))
    la = oracle.decay_gate(np.broadcast_to(f[:, None, None], (50, H, dk)).copy(), A, b)
    assert np.all(la < 0.0) and np.all(np.diff(la[:, 0, 0]) < 0.0)
    # the bias is per (head, channel) and the rate per head
    b2 = b.copy()
    b2[1, 2] = 1.5
    f0 = np.zeros((1, H, dk))
    d = oracle.decay_gate(f0, A, b2) - oracle.decay_gate(f0, A, b)
    assert np.count_nonzero(d) == 1 and d[0, 1, 2] < 0.0
    A2 = A.copy()
    A2[0] += np.log(5.0)
    r = oracle.decay_gate(f0, A2, b) / oracle.decay_gate(f0, A, b)
    assert np.allclose(r[0, 0], 5.0, rtol=1e-14) and np.allclose(r[0, 1], 1.0, rtol=1e-15)


def test_layer_forward_is_invariant_to_positive_rescaling_of_q_and_k():
    """With the normalisation inside, scaling each raw q_t and k_t by any
    positive factor changes nothing (up to the epsilon)."""
    x = gen.make_layer_inputs(1, 70, 2, 16, 16, seed=3)
    rng = np.random.default_rng(4)
    s_q = rng.uniform(0.5, 4.0, (1, 70, 2, 1))
    s_k = rng.uniform(0.5, 4.0, (1, 70, 2, 1))
    args = (x["v"], x["f"], x["A_log"], x["dt_bias"], x["beta"], x["S0"])
    o1, S1 = oracle.forward_layer(x["q"], x["k"], *args, qk_eps=0.0)
    o2, S2 = oracle.forward_layer(x["q"].double().numpy() * s_q, x["k"].double().numpy() * s_k, *args, qk_eps=0.0)
    assert np.allclose(o1, o2, rtol=1e-10, atol=1e-12)
    assert np.allclose(S1, S2, rtol=1e-10, atol=1e-12)


def test_bad_arguments_are_refused():
    with pytest.raises(ValueError):
        oracle.l2norm(np.ones((2, 4)), -1.0)
    with pytest.raises(ValueError):
        oracle.decay_gate(np.ones((1, 2, 4)), np.ones(3), np.ones((2, 4)))
    with pytest.raises(ValueError):
        oracle.decay_gate(np.ones((1, 2, 4)), np.ones(2), np.ones((4, 2)))
