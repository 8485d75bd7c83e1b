"""fp64 CPU oracle for the KDA operator -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library in
``gated_delta_rule_110_b200``) never does; the two share no code.

The arithmetic lives in ``kda_oracle.c`` (plain C, double precision, one token
at a time); this module only compiles it with gcc and marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "kda_oracle.c"
_LIB = _HERE / "libkda_oracle.so"
_lib = None


def build(force: bool = False) -> Path:
    """Compile kda_oracle.c into libkda_oracle.so next to it (gcc, OpenMP)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.tmp{os.getpid()}")
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", str(_SRC), "-o", str(tmp), "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(str(_LIB))
        dp = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        lib.kda_oracle_forward_mut.argtypes = [
            ctypes.c_int, i64p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int,
        ]
        lib.kda_oracle_forward_mut.restype = ctypes.c_int
        lib.kda_oracle_decode.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            dp, dp, dp, dp, dp, dp, dp, ctypes.c_int,
        ]
        lib.kda_oracle_decode.restype = ctypes.c_int
        lib.kda_oracle_mutation_count.restype = ctypes.c_int
        lib.kda_oracle_output_gate.argtypes = [ctypes.c_int64, ctypes.c_int, dp, dp, dp, ctypes.c_double, dp]
        lib.kda_oracle_output_gate.restype = ctypes.c_int
        ip = ctypes.POINTER(ctypes.c_int64)
        lib.kda_oracle_backward.argtypes = [ctypes.c_int, ip, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp]
        lib.kda_oracle_backward.restype = ctypes.c_int
        lib.kda_oracle_l2norm.argtypes = [ctypes.c_int64, ctypes.c_int, dp, ctypes.c_double, dp]
        lib.kda_oracle_l2norm.restype = ctypes.c_int
        lib.kda_oracle_decay_gate.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, dp, dp, dp, dp]
        lib.kda_oracle_decay_gate.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor: take the exact bits it holds
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def mutation_count() -> int:
    return int(_load().kda_oracle_mutation_count())


def forward(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, n_threads: int = 0, mutation: int = 0):
    """Token-by-token KDA forward in fp64.

    Shapes follow the library: either batched ``q,k,log_alpha: [B,T,H,dk]``,
    ``v: [B,T,H,dv]``, ``beta: [B,T,H]`` with ``S0: [B,H,dk,dv]``; or packed
    (``B == 1`` and ``cu_seqlens`` of N+1 offsets) with ``S0: [N,H,dk,dv]``.
    Returns ``(o, S_T)`` as float64 numpy arrays (o shaped like v).
    """
    q, k, v, la, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    if q.ndim != 4:
        raise ValueError("q must be [B, T, H, dk]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        if B != 1:
            raise ValueError("packed input needs B == 1")
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = len(cu) - 1
    s0 = None if S0 is None else _f64(S0).reshape(N, H, dk, dv)
    o = np.zeros((B * T, H, dv))
    ST = np.zeros((N, H, dk, dv))
    rc = _load().kda_oracle_forward_mut(
        N, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), H, dk, dv,
        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b),
        _ptr(s0) if s0 is not None else None, _ptr(o), _ptr(ST), int(n_threads), int(mutation),
    )
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return o.reshape(B, T, H, dv), ST


def decode(q, k, v, log_alpha, beta, S, n_threads: int = 0):
    """One recurrent step for ``[N, H, d]`` inputs; returns ``(o, S_new)``."""
    q, k, v, la, b, S = (_f64(x) for x in (q, k, v, log_alpha, beta, S))
    N, H, dk = q.shape
    dv = v.shape[-1]
    S = S.copy()
    o = np.zeros((N, H, dv))
    rc = _load().kda_oracle_decode(N, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b),
                                   _ptr(S), _ptr(o), int(n_threads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return o, S


def output_gate(o, g, w, eps: float):
    """Per-head RMSNorm with weight ``w`` ([dv]) and sigmoid output gate ``g``
    (same shape as ``o``, last axis dv), in fp64; returns an array shaped like o."""
    o, g, w = _f64(o), _f64(g), _f64(w)
    if o.shape != g.shape or w.shape != (o.shape[-1],):
        raise ValueError("o and g must match; w must have dv values")
    dv = o.shape[-1]
    out = np.zeros_like(o)
    rc = _load().kda_oracle_output_gate(o.size // dv, dv, _ptr(o), _ptr(g), _ptr(w), float(eps), _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out


def l2norm(x, eps: float):
    """x / sqrt(sum(x^2) + eps) over the last axis, in fp64 (the L2
    normalisation of q and k); returns an array shaped like x."""
    x = _f64(x)
    d = x.shape[-1]
    out = np.zeros_like(x)
    if _load().kda_oracle_l2norm(x.size // d, d, _ptr(x), float(eps), _ptr(out)) != 0:
        raise ValueError("oracle rejected its arguments")
    return out


def decay_gate(f, A_log, dt_bias):
    """log alpha = -exp(A_log[h]) * softplus(f + dt_bias[h, c]) in fp64.
    f: [..., H, dk]; A_log: [H]; dt_bias: [H, dk]."""
    f, A_log, dt_bias = _f64(f), _f64(A_log), _f64(dt_bias)
    H, dk = f.shape[-2], f.shape[-1]
    if A_log.shape != (H,) or dt_bias.shape != (H, dk):
        raise ValueError("A_log must be [H] and dt_bias [H, dk]")
    out = np.zeros_like(f)
    if _load().kda_oracle_decay_gate(f.size // (H * dk), H, dk, _ptr(f), _ptr(A_log), _ptr(dt_bias), _ptr(out)) != 0:
        raise ValueError("oracle rejected its arguments")
    return out


def forward_layer(q, k, v, f, A_log, dt_bias, beta, S0=None, cu_seqlens=None, qk_eps: float = 1e-6,
                  out_gate=None, norm_weight=None, eps: float = 1e-5):
    """The operator with the layer's producer and (optionally) consumer steps,
    composed from the functions above: forward(l2norm(q), l2norm(k), v,
    decay_gate(f, A_log, dt_bias), beta, S0), then output_gate when out_gate
    is given.  Returns (o, S_T)."""
    o, S = forward(l2norm(q, qk_eps), l2norm(k, qk_eps), v, decay_gate(f, A_log, dt_bias), beta, S0,
                   cu_seqlens=cu_seqlens)
    if out_gate is not None:
        o = output_gate(o, out_gate, norm_weight, eps)
    return o, S


def backward(q, k, v, log_alpha, beta, S0=None, dO=None, dS_T=None, cu_seqlens=None):
    """Gradients of the operator in fp64 by hand-written reverse-mode
    differentiation of the token recurrence (kda_oracle.c,
    kda_oracle_backward).  Shapes as forward; dO like o, dS_T like S_T.
    Returns (dq, dk, dv, dlog_alpha, dbeta, dS0)."""
    q, k, v, la, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        if B != 1:
            raise ValueError("packed input needs B == 1")
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = len(cu) - 1
    s0 = None if S0 is None else _f64(S0).reshape(N, H, dk, dv)
    gO = None if dO is None else _f64(dO).reshape(B * T, H, dv)
    gS = None if dS_T is None else _f64(dS_T).reshape(N, H, dk, dv)
    dq, dk_, dla = (np.zeros((B * T, H, dk)) for _ in range(3))
    dv_ = np.zeros((B * T, H, dv))
    db = np.zeros((B * T, H))
    dS0 = np.zeros((N, H, dk, dv))
    opt = lambda a: _ptr(a) if a is not None else None
    rc = _load().kda_oracle_backward(
        N, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(la),
        _ptr(b), opt(s0), opt(gO), opt(gS), _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dla), _ptr(db), _ptr(dS0))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    r = lambda a, last: a.reshape(B, T, H, *last)
    return (r(dq, (dk,)), r(dk_, (dk,)), r(dv_, (dv,)), r(dla, (dk,)), db.reshape(B, T, H), dS0)
