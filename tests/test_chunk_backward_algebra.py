"""The chunkwise form of the operator's gradients, derived here for a
tensor-core backward and checked in fp64 against the oracle's token-by-token
gradients (oracle.backward, itself pinned by finite differences).

Forward of one chunk (C rows, state S at its start; g = per-channel cumulative
log decay inside the chunk, gamma = g of its last row; the chunkwise section of
the "Kimi Linear" summary gives this structure: UT transform, intra- plus
inter-chunk output):
    Kd = k o e^g,  Qd = q o e^g,  Ki = k o e^-g,  Kh = k o e^(gamma - g)
    A  = strict_tril(Diag(beta) Kd Ki^T),   T = (I + A)^-1
    R  = V - Kd S,   U = T Diag(beta) R
    O  = Qd S + P U,  P = tril(Qd Ki^T)
    S' = Diag(e^gamma) S + Kh^T U
Backward, given dO and dS' (reverse of each line above):
    dS  = Diag(e^gamma) dS' + Qd^T dO - Kd^T dR
    dU  = Kh dS' + P^T dO,   dKh = U dS'^T,   dP = tril(dO U^T),   dQd = dO S^T + dP Ki
    dX  = T^T dU  (X = Diag(beta) R),   dA = -strict_tril(dX U^T)
    dR  = Diag(beta) dX,   dV = dR,   dKd = -dR S^T + Diag(beta) dA Ki
    dKi = (Diag(beta) dA)^T Kd + dP^T Qd
    dbeta = rowsum(dX o R) + rowsum(dA o (Kd Ki^T))
    dk  = dKd o e^g + dKi o e^-g + dKh o e^(gamma - g),   dq = dQd o e^g
    dg  = dKd o Kd + dQd o Qd - dKi o Ki - dKh o Kh,  plus  e^gamma o rowsum(dS' o S) + colsum(dKh o Kh) on the last row
    dlog_alpha = reverse cumulative sum of dg over the chunk's rows
The state gradient dS goes to the previous chunk.  (Plain exponentials: the
kernel would use the forward's per-chunk reference point; moderate decays
here keep fp64 exact enough for the comparison.)
"""
import numpy as np
import pytest

import oracle


def _chunk_backward(q, k, v, la, beta, S0, dO, dST, C):
    """One (sequence, head): inputs [T, d]; returns (dq, dk, dv, dla, dbeta, dS0)."""
    T, dk = q.shape
    n_chunks = (T + C - 1) // C
    # forward, keeping each chunk's initial state
    S = S0.copy()
    starts = []
    for c in range(n_chunks):
        a, e = c * C, min(T, (c + 1) * C)
        starts.append(S.copy())
        g = np.cumsum(la[a:e], axis=0)
        gam = g[-1]
        Kd, Qd, Ki, Kh = k[a:e] * np.exp(g), q[a:e] * np.exp(g), k[a:e] * np.exp(-g), k[a:e] * np.exp(gam - g)
        A = np.tril(beta[a:e, None] * (Kd @ Ki.T), -1)
        Tm = np.linalg.inv(np.eye(e - a) + A)
        U = Tm @ (beta[a:e, None] * (v[a:e] - Kd @ S))
        S = np.exp(gam)[:, None] * S + Kh.T @ U
    grads = [np.zeros_like(x) for x in (q, k, v, la)] + [np.zeros_like(beta)]
    dq, dk_, dv, dla, dbeta = grads
    dS = dST.copy()
    for c in reversed(range(n_chunks)):
        a, e = c * C, min(T, (c + 1) * C)
        S = starts[c]
        g = np.cumsum(la[a:e], axis=0)
        gam = g[-1]
        b = beta[a:e]
        Kd, Qd, Ki, Kh = k[a:e] * np.exp(g), q[a:e] * np.exp(g), k[a:e] * np.exp(-g), k[a:e] * np.exp(gam - g)
        KK = Kd @ Ki.T
        A = np.tril(b[:, None] * KK, -1)
        Tm = np.linalg.inv(np.eye(e - a) + A)
        R = v[a:e] - Kd @ S
        U = Tm @ (b[:, None] * R)
        P = np.tril(Qd @ Ki.T)
        dSn, dOc = dS, dO[a:e]
        dU = Kh @ dSn + P.T @ dOc
        dKh = U @ dSn.T
        dP = np.tril(dOc @ U.T)
        dQd = dOc @ S.T + dP @ Ki
        dX = Tm.T @ dU
        dA = -np.tril(dX @ U.T, -1)
        dR = b[:, None] * dX
        dKd = -dR @ S.T + (b[:, None] * dA) @ Ki
        dKi = (b[:, None] * dA).T @ Kd + dP.T @ Qd
        dbeta[a:e] = np.sum(dX * R, axis=1) + np.sum(dA * KK, axis=1)
        dv[a:e] = dR
        dk_[a:e] = dKd * np.exp(g) + dKi * np.exp(-g) + dKh * np.exp(gam - g)
        dq[a:e] = dQd * np.exp(g)
        dg = dKd * Kd + dQd * Qd - dKi * Ki - dKh * Kh
        dg[-1] += np.exp(gam) * np.sum(dSn * S, axis=1) + np.sum(dKh * Kh, axis=0)
        dla[a:e] = np.cumsum(dg[::-1], axis=0)[::-1]
        dS = np.exp(gam)[:, None] * dSn + Qd.T @ dOc - Kd.T @ dR
    return dq, dk_, dv, dla, dbeta, dS


@pytest.mark.parametrize("T,C", [(37, 8), (64, 16), (5, 8)])
def test_chunk_backward_equals_token_backward(T, C):
    rng = np.random.default_rng(T + C)
    dk, dv = 6, 5
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk)) / np.sqrt(dk)
    v = rng.standard_normal((T, dv))
    la = -rng.uniform(0.01, 0.4, (T, dk))
    beta = rng.uniform(0.1, 1.0, T)
    S0 = rng.standard_normal((dk, dv)) * 0.5
    dO = rng.standard_normal((T, dv))
    dST = rng.standard_normal((dk, dv))
    ref = oracle.backward(q[None, :, None], k[None, :, None], v[None, :, None], la[None, :, None],
                          beta[None, :, None], S0[None, None], dO=dO[None, :, None], dS_T=dST[None, None])
    ref = [r[0, :, 0] for r in ref[:5]] + [ref[5][0, 0]]
    got = _chunk_backward(q, k, v, la, beta, S0, dO, dST, C)
    for name, a, b in zip(("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"), got, ref):
        assert np.allclose(a, b, rtol=1e-9, atol=1e-11), name
