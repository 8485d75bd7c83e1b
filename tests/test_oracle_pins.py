"""Pins of the fp64 oracle to what the pages and the mathematics fix.

The oracle (``oracle/kda_oracle.c``) runs the KDA recurrence token by token.
None of these checks re-types its loop: each compares it with a different
formulation -- dense transition-matrix products, an autograd gradient step,
closed forms, Householder identities, structural invariances -- chosen so that
a plausible slip in the oracle (decay applied after the delta step, output
from the pre-update state, a transposed read-out, a sign error, beta dropped
from the erase term, the gate on the wrong axis, S0 ignored, the error term
computed from the undecayed state) fails at least one of them.  The last test
plants each of those slips in the oracle and checks exactly that.

Sources (page titles and sections):
  "Kimi Linear" summary (pt.news.hada.io; the Vietnamese copy on
  vi.news.hada.io says the same):
    - "Da atencao linear ao Gated DeltaNet": DeltaNet is online gradient
      descent on the reconstruction loss; the rank-1 update is a generalised
      Householder transform; GDN adds a scalar forget gate.
    - "Controle fino de memoria no Kimi Delta Attention": the scalar gate
      becomes a per-channel (per key dimension) diagonal gate.
    - "Algoritmo paralelo por chunks": the final state of a chunk is the
      initial state of the next (split/resume invariance).
"""
import numpy as np
import pytest
import torch

import oracle

RNG = np.random.default_rng(1234)


def rand_case(T, H, dk, dv, *, B=1, beta_scale=1.0, gate=0.3, seed=0, s0=True):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, T, H, dk))
    k = r.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((B, T, H, dv))
    la = -gate * np.log1p(np.exp(r.standard_normal((B, T, H, dk))))
    beta = beta_scale / (1 + np.exp(-r.standard_normal((B, T, H))))
    S0 = r.standard_normal((B, H, dk, dv)) * 0.5 if s0 else None
    return q, k, v, la, beta, S0


def brute_force(q, k, v, la, beta, S0):
    """Dense transition products for one (sequence, head).

    M_t = (I - beta_t k_t k_t^T) Diag(exp(la_t)); with P_{a..b} = M_b ... M_a:
        S_t = P_{1..t} S0 + sum_{s<=t} P_{s+1..t} beta_s k_s v_s^T
        o_t = S_t^T q_t
    q, k, la: [T, dk]; v: [T, dv]; beta: [T]; S0: [dk, dv] (or None).
    """
    T, dk = k.shape
    dv = v.shape[1]
    S0 = np.zeros((dk, dv)) if S0 is None else S0
    M = [(np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(la[t])) for t in range(T)]
    o = np.zeros((T, dv))
    S_t = None
    for t in range(T):
        P = np.eye(dk)
        for s in range(t + 1):
            P = M[s] @ P
        S_t = P @ S0
        for s in range(t + 1):
            Ps = np.eye(dk)
            for u in range(s + 1, t + 1):
                Ps = M[u] @ Ps
            S_t = S_t + Ps @ (beta[s] * np.outer(k[s], v[s]))
        o[t] = S_t.T @ q[t]
    return o, (S_t if S_t is not None else S0.copy())


def run(q, k, v, la, beta, S0, mutation=0, cu=None):
    return oracle.forward(q, k, v, la, beta, S0, cu_seqlens=cu, mutation=mutation)


# ---------------------------------------------------------------------------
# 0. A worked example computed by hand (dk = dv = 2, T = 2, S0 = 0)
# ---------------------------------------------------------------------------
def test_hand_worked_example():
    # t=1: k=(1,0) v=(2,4) q=(1,1) beta=1/2 alpha=(1,1)
    #      S~=0, kS=0, d=(1,2), S1=[[1,2],[0,0]], o1=S1^T q=(1,2)
    # t=2: k=(0.6,0.8) v=(1,-1) q=(0,1) beta=1 alpha=(0.5,1)
    #      S~=[[0.5,1],[0,0]], kS=S~^T k=(0.3,0.6), d=(0.7,-1.6)
    #      S2=S~ + k d^T=[[0.92,0.04],[0.56,-1.28]], o2=S2^T q=(0.56,-1.28)
    q = np.array([[1.0, 1.0], [0.0, 1.0]]).reshape(1, 2, 1, 2)
    k = np.array([[1.0, 0.0], [0.6, 0.8]]).reshape(1, 2, 1, 2)
    v = np.array([[2.0, 4.0], [1.0, -1.0]]).reshape(1, 2, 1, 2)
    la = np.array([[0.0, 0.0], [np.log(0.5), 0.0]]).reshape(1, 2, 1, 2)
    beta = np.array([0.5, 1.0]).reshape(1, 2, 1)
    o, S = run(q, k, v, la, beta, None)
    np.testing.assert_allclose(o.reshape(2, 2), [[1.0, 2.0], [0.56, -1.28]], atol=1e-14)
    np.testing.assert_allclose(S.reshape(2, 2), [[0.92, 0.04], [0.56, -1.28]], atol=1e-14)


# ---------------------------------------------------------------------------
# 1. Brute force: explicit transition-matrix products on tiny inputs
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T,dk,dv", [(1, 3, 5), (5, 4, 3), (8, 6, 7), (7, 5, 5)])
def test_brute_force_transition_products(T, dk, dv):
    q, k, v, la, beta, S0 = rand_case(T, 2, dk, dv, seed=T * 31 + dk)
    o, ST = run(q, k, v, la, beta, S0)
    for h in range(2):
        ob, Sb = brute_force(q[0, :, h], k[0, :, h], v[0, :, h], la[0, :, h], beta[0, :, h], S0[0, h])
        np.testing.assert_allclose(o[0, :, h], ob, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(ST[0, h], Sb, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------
# 2. alpha == 1: DeltaNet = online SGD on 1/2 ||S^T k - v||^2 (autograd)
# ---------------------------------------------------------------------------
def deltanet_sgd(k, v, beta, S0):
    S = torch.tensor(S0, dtype=torch.float64)
    out = []
    for t in range(k.shape[0]):
        S = S.detach().requires_grad_(True)
        kt = torch.tensor(k[t])
        vt = torch.tensor(v[t])
        loss = 0.5 * ((S.T @ kt - vt) ** 2).sum()
        (grad,) = torch.autograd.grad(loss, S)
        S = (S - float(beta[t]) * grad).detach()
        out.append(S.clone())
    return [s.numpy() for s in out]


def test_deltanet_is_online_gradient_descent():
    T, dk, dv = 9, 6, 4
    q, k, v, la, beta, S0 = rand_case(T, 1, dk, dv, seed=7)
    la[:] = 0.0
    o, ST = run(q, k, v, la, beta, S0)
    states = deltanet_sgd(k[0, :, 0], v[0, :, 0], beta[0, :, 0], S0[0, 0])
    np.testing.assert_allclose(ST[0, 0], states[-1], rtol=1e-12, atol=1e-12)
    for t in range(T):
        np.testing.assert_allclose(o[0, t, 0], states[t].T @ q[0, t, 0], rtol=1e-12, atol=1e-12)


def test_deltanet_step_lowers_reconstruction_loss():
    # with ||k|| = 1 and 0 < beta < 2 one step strictly lowers 1/2||S^T k - v||^2
    T, dk, dv = 6, 5, 3
    q, k, v, la, beta, S0 = rand_case(T, 1, dk, dv, seed=8)
    la[:] = 0.0
    S = S0[0, 0]
    for t in range(T):
        before = 0.5 * np.sum((S.T @ k[0, t, 0] - v[0, t, 0]) ** 2)
        _, S_next = run(q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1], la[:, t:t + 1],
                        beta[:, t:t + 1], S[None, None])
        S = S_next[0, 0]
        after = 0.5 * np.sum((S.T @ k[0, t, 0] - v[0, t, 0]) ** 2)
        assert after < before
        # closed form of the shrink factor: (1 - beta)^2
        np.testing.assert_allclose(after, before * (1 - beta[0, t, 0]) ** 2, rtol=1e-10)


# ---------------------------------------------------------------------------
# 3. gate constant across channels: Gated DeltaNet with a scalar gate
# ---------------------------------------------------------------------------
def test_scalar_gate_reduces_to_gated_deltanet():
    T, dk, dv = 10, 5, 6
    q, k, v, la, beta, S0 = rand_case(T, 1, dk, dv, seed=9)
    la[:] = la[..., :1]  # one gate value per (token, head)
    o, ST = run(q, k, v, la, beta, S0)
    S = S0[0, 0].copy()
    for t in range(T):
        a = np.exp(la[0, t, 0, 0])
        kt = k[0, t, 0]
        # GDN: S_t = a_t (I - beta k k^T) S_{t-1} + beta k v^T
        S = a * (np.eye(dk) - beta[0, t, 0] * np.outer(kt, kt)) @ S + beta[0, t, 0] * np.outer(kt, v[0, t, 0])
        np.testing.assert_allclose(o[0, t, 0], S.T @ q[0, t, 0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ST[0, 0], S, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# 4. beta == 0: pure per-channel decay (closed form)
# ---------------------------------------------------------------------------
def test_beta_zero_closed_form():
    T, dk, dv = 12, 7, 5
    q, k, v, la, beta, S0 = rand_case(T, 2, dk, dv, seed=10, gate=2.0)
    beta[:] = 0.0
    o, ST = run(q, k, v, la, beta, S0)
    g = np.cumsum(la, axis=1)  # [B, T, H, dk]
    for h in range(2):
        np.testing.assert_allclose(ST[0, h], np.exp(g[0, -1, h])[:, None] * S0[0, h], rtol=1e-12)
        for t in range(T):
            ref = S0[0, h].T @ (q[0, t, h] * np.exp(g[0, t, h]))
            np.testing.assert_allclose(o[0, t, h], ref, rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------------------
# 5. Householder identities (unit-norm keys)
# ---------------------------------------------------------------------------
def test_beta_one_memorises_exactly():
    # beta = 1, ||k|| = 1: k^T S_t = v_t^T; read with q = k it returns v
    T, dk, dv = 10, 6, 4
    q, k, v, la, beta, S0 = rand_case(T, 1, dk, dv, seed=11)
    beta[:] = 1.0
    o, _ = run(k, k, v, la, beta, S0)
    np.testing.assert_allclose(o, v, rtol=1e-12, atol=1e-12)


def test_general_beta_projection_identity():
    # ||k|| = 1: k^T S_t = (1 - beta) k^T Diag(alpha) S_{t-1} + beta v^T
    T, dk, dv = 8, 5, 3
    q, k, v, la, beta, S0 = rand_case(T, 1, dk, dv, seed=12, beta_scale=1.7)
    o, _ = run(k, k, v, la, beta, S0)
    S_prev = S0[0, 0]
    for t in range(T):
        St = np.exp(la[0, t, 0])[:, None] * S_prev
        ref = (1 - beta[0, t, 0]) * (St.T @ k[0, t, 0]) + beta[0, t, 0] * v[0, t, 0]
        np.testing.assert_allclose(o[0, t, 0], ref, rtol=1e-11, atol=1e-12)
        _, S_prev = run(q[:, :t + 1], k[:, :t + 1], v[:, :t + 1], la[:, :t + 1], beta[:, :t + 1], S0)
        S_prev = S_prev[0, 0]


def test_beta_two_is_a_reflection():
    # beta = 2, alpha = 1, v = 0: S <- (I - 2 k k^T) S, an orthogonal map
    T, dk, dv = 9, 6, 5
    q, k, v, la, beta, S0 = rand_case(T, 1, dk, dv, seed=13)
    beta[:] = 2.0
    la[:] = 0.0
    v[:] = 0.0
    _, ST = run(q, k, v, la, beta, S0)
    np.testing.assert_allclose(np.linalg.norm(ST), np.linalg.norm(S0), rtol=1e-12)
    # and applying the reflections in reverse order undoes them
    S = ST[0, 0]
    for t in reversed(range(T)):
        kt = k[0, t, 0]
        S = (np.eye(dk) - 2 * np.outer(kt, kt)) @ S
    np.testing.assert_allclose(S, S0[0, 0], rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------
# 6. Structure
# ---------------------------------------------------------------------------
def test_linear_in_values_and_initial_state():
    T, dk, dv = 11, 4, 6
    q, k, v1, la, beta, S01 = rand_case(T, 2, dk, dv, seed=14)
    _, _, v2, _, _, S02 = rand_case(T, 2, dk, dv, seed=15)
    a, b = 0.7, -1.3
    o1, S1 = run(q, k, v1, la, beta, S01)
    o2, S2 = run(q, k, v2, la, beta, S02)
    o, S = run(q, k, a * v1 + b * v2, la, beta, a * S01 + b * S02)
    np.testing.assert_allclose(o, a * o1 + b * o2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S, a * S1 + b * S2, rtol=1e-11, atol=1e-12)


def test_value_column_permutation_commutes():
    T, dk, dv = 9, 5, 7
    q, k, v, la, beta, S0 = rand_case(T, 2, dk, dv, seed=16)
    perm = np.random.default_rng(3).permutation(dv)
    o, S = run(q, k, v, la, beta, S0)
    op, Sp = run(q, k, v[..., perm], la, beta, S0[..., perm])
    np.testing.assert_allclose(op, o[..., perm], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(Sp, S[..., perm], rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("T1", [1, 5, 13])
def test_split_resume(T1):
    T, dk, dv = 20, 6, 5
    q, k, v, la, beta, S0 = rand_case(T, 2, dk, dv, seed=17)
    o, S = run(q, k, v, la, beta, S0)
    oa, Sa = run(q[:, :T1], k[:, :T1], v[:, :T1], la[:, :T1], beta[:, :T1], S0)
    ob, Sb = run(q[:, T1:], k[:, T1:], v[:, T1:], la[:, T1:], beta[:, T1:], Sa)
    np.testing.assert_allclose(np.concatenate([oa, ob], axis=1), o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(Sb, S, rtol=1e-12, atol=1e-13)


def test_packed_varlen_equals_separate_runs_and_heads_independent():
    lens = [3, 0, 9, 1, 6]
    H, dk, dv = 3, 5, 4
    Ttot = sum(lens)
    q, k, v, la, beta, _ = rand_case(Ttot, H, dk, dv, seed=18)
    S0 = np.random.default_rng(5).standard_normal((len(lens), H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lens)])
    o, S = run(q, k, v, la, beta, S0, cu=cu)
    for n, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        on, Sn = run(q[:, a:b], k[:, a:b], v[:, a:b], la[:, a:b], beta[:, a:b], S0[n:n + 1])
        np.testing.assert_allclose(o[:, a:b], on, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(S[n], Sn[0], rtol=1e-13, atol=1e-14)
    # empty sequence: final state equals initial state
    np.testing.assert_array_equal(S[1], S0[1])
    # perturbing head 2 leaves heads 0 and 1 untouched
    v2 = v.copy()
    v2[..., 2, :] += 1.0
    o2, S2 = run(q, k, v2, la, beta, S0, cu=cu)
    np.testing.assert_array_equal(o2[..., :2, :], o[..., :2, :])
    np.testing.assert_array_equal(S2[:, :2], S[:, :2])


def test_decode_steps_equal_forward():
    T, H, dk, dv = 6, 2, 5, 4
    q, k, v, la, beta, S0 = rand_case(T, H, dk, dv, seed=19)
    o, S = run(q, k, v, la, beta, S0)
    Sd = S0[0].copy()[None]  # [N=1, H, dk, dv]
    for t in range(T):
        od, Sd = oracle.decode(q[:, t], k[:, t], v[:, t], la[:, t], beta[:, t], Sd)
        np.testing.assert_allclose(od, o[:, t], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(Sd, S, rtol=1e-13, atol=1e-14)


def test_threads_do_not_change_bits():
    q, k, v, la, beta, S0 = rand_case(30, 4, 6, 6, B=3, seed=20)
    a = oracle.forward(q, k, v, la, beta, S0, n_threads=1)
    b = oracle.forward(q, k, v, la, beta, S0, n_threads=4)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


# ---------------------------------------------------------------------------
# 7. Pin strength: every planted slip fails some pin above
# ---------------------------------------------------------------------------
def _pins_failing(mutation):
    """Cheap versions of the pins above, run against a mutated oracle."""
    failed = []

    def m(*args, cu=None):
        return oracle.forward(*args, cu_seqlens=cu, mutation=mutation)

    # brute force (dk == dv so the transposed read-out is defined)
    q, k, v, la, beta, S0 = rand_case(6, 1, 5, 5, seed=101)
    o, S = m(q, k, v, la, beta, S0)
    ob, Sb = brute_force(q[0, :, 0], k[0, :, 0], v[0, :, 0], la[0, :, 0], beta[0, :, 0], S0[0, 0])
    if not (np.allclose(o[0, :, 0], ob, atol=1e-10) and np.allclose(S[0, 0], Sb, atol=1e-10)):
        failed.append("brute_force")
    # memorisation with beta = 1 (q = k)
    beta1 = np.ones_like(beta)
    o, _ = m(k, k, v, la, beta1, S0)
    if not np.allclose(o, v, atol=1e-10):
        failed.append("memorise")
    # beta = 0 closed form
    beta0 = np.zeros_like(beta)
    o, S = m(q, k, v, la, beta0, S0)
    g = np.cumsum(la, axis=1)
    if not np.allclose(S[0, 0], np.exp(g[0, -1, 0])[:, None] * S0[0, 0], atol=1e-10):
        failed.append("beta_zero")
    # DeltaNet SGD (alpha = 1)
    la0 = np.zeros_like(la)
    _, S = m(q, k, v, la0, beta, S0)
    st = deltanet_sgd(k[0, :, 0], v[0, :, 0], beta[0, :, 0], S0[0, 0])
    if not np.allclose(S[0, 0], st[-1], atol=1e-10):
        failed.append("deltanet")
    return failed


def test_every_planted_slip_is_caught():
    assert _pins_failing(0) == []
    for mutation in range(1, oracle.mutation_count()):
        assert _pins_failing(mutation), f"planted slip {mutation} passed every pin"


def test_golden_regression_fixture():
    import json
    from pathlib import Path
    d = json.loads((Path(__file__).parent / "golden" / "oracle_tiny.json").read_text())
    arr = {k: np.array(v) for k, v in d.items()}
    o, S = oracle.forward(arr["q"], arr["k"], arr["v"], arr["log_alpha"], arr["beta"], arr["S0"])
    np.testing.assert_allclose(o, arr["o"], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(S, arr["S_T"], rtol=1e-14, atol=1e-15)
