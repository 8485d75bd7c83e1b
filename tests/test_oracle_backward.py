"""Pins of the oracle's gradients (oracle.backward): every partial derivative
of a random linear functional of (o, S_T) against central finite differences
of oracle.forward in fp64, on tiny packed and batched inputs.  The forward is
pinned on its own (test_oracle_pins.py); finite differences use nothing but
it, so a slip anywhere in the hand-written reverse pass fails here."""
import numpy as np
import pytest

import oracle


def _inputs(rng, B, T, H, dk, dv, packed):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk)) * 0.6
    v = rng.standard_normal((B, T, H, dv))
    la = -rng.uniform(0.05, 1.5, (B, T, H, dk))
    beta = rng.uniform(0.1, 1.0, (B, T, H))
    N = len(packed) if packed else B
    S0 = rng.standard_normal((N, H, dk, dv)) * 0.3
    cu = None
    if packed:
        cu = np.concatenate([[0], np.cumsum(packed)]).astype(np.int64)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=beta, S0=S0, cu=cu)


def _loss(x, R1, R2):
    o, S = oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], cu_seqlens=x["cu"])
    return float(np.sum(o * R1) + np.sum(S * R2))


@pytest.mark.parametrize("B,T,packed", [(1, 7, [3, 0, 4]), (2, 4, None)])
def test_gradients_match_central_differences(B, T, packed):
    rng = np.random.default_rng(11 + B)
    H, dk, dv = 2, 3, 2
    x = _inputs(rng, B, T, H, dk, dv, packed)
    o, S = oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], cu_seqlens=x["cu"])
    R1 = rng.standard_normal(o.shape)
    R2 = rng.standard_normal(S.shape)
    grads = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], dO=R1, dS_T=R2,
                            cu_seqlens=x["cu"])
    eps = 1e-6
    for name, g in zip(("q", "k", "v", "log_alpha", "beta", "S0"), grads):
        assert g.shape == x[name].shape, name
        it = np.nditer(x[name], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            keep = x[name][idx]
            x[name][idx] = keep + eps
            lp = _loss(x, R1, R2)
            x[name][idx] = keep - eps
            lm = _loss(x, R1, R2)
            x[name][idx] = keep
            fd = (lp - lm) / (2 * eps)
            assert abs(g[idx] - fd) <= 1e-6 * max(1.0, abs(fd)), f"d{name}{idx}: {g[idx]} vs {fd}"


def test_no_upstream_gradient_gives_zero():
    rng = np.random.default_rng(3)
    x = _inputs(rng, 1, 5, 1, 3, 2, None)
    grads = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    assert all(np.all(g == 0.0) for g in grads)


def test_final_state_gradient_only_through_the_last_token_of_a_one_token_sequence():
    """One token, dO = 0, dS_T = G: S_T = S~ + beta k u^T, so dS0 =
    Diag(alpha)(G - beta k k^T G) (the transition's transpose applied to G)."""
    rng = np.random.default_rng(4)
    x = _inputs(rng, 1, 1, 1, 4, 3, None)
    G = rng.standard_normal((1, 1, 4, 3))
    *_, dS0 = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], dS_T=G)
    k = x["k"][0, 0, 0]
    b = x["beta"][0, 0, 0]
    alpha = np.exp(x["log_alpha"][0, 0, 0])
    ref = np.diag(alpha) @ (np.eye(4) - b * np.outer(k, k)) @ G[0, 0]
    assert np.allclose(dS0[0, 0], ref, rtol=1e-13, atol=1e-15)
