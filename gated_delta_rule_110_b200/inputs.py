"""Seeded synthetic inputs for the KDA operator.

This module holds the input *distributions* only -- none of the operator's
arithmetic -- so that the CUDA path and the fp64 oracle can both be fed the
exact same bits.  Every tensor comes from a ``torch.Generator`` seeded from the
workload's seed, on the device asked for.

Workloads (sizes and value distributions of the benchmark configurations):

=========  =========================================================  ======
name       shape                                                      dtype
=========  =========================================================  ======
oracle     B=1, H=2, T=256, dk=dv=64, C=64                            fp32
prefill    B=4, H=16, T=4096, dk=dv=128, C=64                         bf16
varlen     8 sequences, lengths ~ U{512..8192}, H=32, dk=dv=128       bf16
long       B=1, H=32, T=131072, dk=dv=128                             bf16
decode     256 sequences x H=32, dk=dv=128, fp32 state, 1000 steps    bf16
=========  =========================================================  ======

Distributions: q, k ~ N(0,1) then L2-normalised per (token, head);
v ~ N(0,1); beta = sigmoid(N(0,1)).  log_alpha:

* ``small``  : -0.1 * softplus(N(0,1))                       (oracle workload)
* ``wide``   : clamp(-exp(U(-5,0)) * softplus(N(0,1)), -5, 0)  (prefill,
               varlen, decode)
* ``long``   : per (head, channel) a mean decay a ~ U(0.9, 0.9999); per token
               log_alpha = log(a) * m_t with m_t ~ U(0.5, 1.5), clamped to
               [-5, 0]                                          (long)

S0 is zero (``small``) or N(0, 0.01) i.e. standard deviation 0.1 (others).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import math

import torch


@dataclass
class Workload:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    chunk: int
    dtype: torch.dtype
    gate: str = "wide"
    s0: str = "normal"
    seqlens: list | None = field(default=None)
    seed: int = 0


BASE_SEED = 20251030


def _varlen_lengths(n: int, lo: int, hi: int, seed: int) -> list:
    g = torch.Generator().manual_seed(seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


def workload(name: str) -> Workload:
    """The named benchmark workload (see the module docstring)."""
    if name == "oracle":
        return Workload("oracle", 1, 256, 2, 64, 64, 64, torch.float32, gate="small", s0="zero",
                        seed=BASE_SEED + 0)
    if name == "prefill":
        return Workload("prefill", 4, 4096, 16, 128, 128, 64, torch.bfloat16, seed=BASE_SEED + 1)
    if name == "varlen":
        lens = _varlen_lengths(8, 512, 8192, BASE_SEED + 2)
        return Workload("varlen", 1, sum(lens), 32, 128, 128, 64, torch.bfloat16, seqlens=lens,
                        seed=BASE_SEED + 2)
    if name == "long":
        return Workload("long", 1, 131072, 32, 128, 128, 64, torch.bfloat16, gate="long",
                        seed=BASE_SEED + 3)
    if name == "decode":
        return Workload("decode", 256, 1, 32, 128, 128, 64, torch.bfloat16, seed=BASE_SEED + 4)
    raise KeyError(name)


def _normal(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def _l2n(x):
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def gate_values(kind: str, T: int, H: int, dk: int, g, device, lead=()):
    """log_alpha of shape lead + (T, H, dk) in fp32 for the named distribution."""
    shape = tuple(lead) + (T, H, dk)
    if kind == "small":
        return -0.1 * torch.nn.functional.softplus(_normal(shape, g, device))
    if kind == "wide":
        u = torch.rand(shape, generator=g, device=device) * 5.0 - 5.0
        sp = torch.nn.functional.softplus(_normal(shape, g, device))
        return (-torch.exp(u) * sp).clamp(-5.0, 0.0)
    if kind == "long":
        a = 0.9 + torch.rand(tuple(lead) + (1, H, dk), generator=g, device=device) * (0.9999 - 0.9)
        m = 0.5 + torch.rand(tuple(lead) + (T, H, 1), generator=g, device=device)
        return (torch.log(a) * m).clamp(-5.0, 0.0)
    if kind == "zero":
        return torch.zeros(shape, device=device)
    raise KeyError(kind)


def make_inputs(B: int, T: int, H: int, dk: int, dv: int, *, dtype=torch.bfloat16,
                gate_dtype=None, gate: str = "wide", s0: str = "normal", seqlens=None,
                seed: int = 0, device="cpu") -> dict:
    """Seeded inputs of the given sizes.

    Returns a dict with q, k, v, log_alpha, beta (dtype / gate_dtype), S0
    (fp32 or None) and cu_seqlens (int32 or None).  With ``seqlens`` the batch
    is packed: B must be 1 and T == sum(seqlens).
    """
    gate_dtype = dtype if gate_dtype is None else gate_dtype
    g = torch.Generator(device=device).manual_seed(seed)
    if seqlens is not None:
        if B != 1 or T != sum(seqlens):
            raise ValueError("packed inputs need B == 1 and T == sum(seqlens)")
        N = len(seqlens)
    else:
        N = B
    q = _l2n(_normal((B, T, H, dk), g, device)).to(dtype)
    k = _l2n(_normal((B, T, H, dk), g, device)).to(dtype)
    v = _normal((B, T, H, dv), g, device).to(dtype)
    beta = torch.sigmoid(_normal((B, T, H), g, device)).to(gate_dtype)
    la = gate_values(gate, T, H, dk, g, device, lead=(B,)).to(gate_dtype)
    if s0 == "zero":
        S0 = torch.zeros((N, H, dk, dv), device=device)
    elif s0 == "none":
        S0 = None
    else:
        S0 = 0.1 * _normal((N, H, dk, dv), g, device)
    cu = None
    if seqlens is not None:
        cu = torch.zeros(N + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(seqlens, dtype=torch.int64), 0).to(torch.int32)
        cu = cu.to(device)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=beta, S0=S0, cu_seqlens=cu)


def output_gate_inputs(v_shape, *, dtype=torch.bfloat16, scale: float = 2.0, seed: int = 0,
                       device="cpu"):
    """Inputs of the fused output epilogue: the gate's pre-activation g (shaped
    like v, normal with standard deviation ``scale``, in ``dtype``) and the
    per-channel RMSNorm weight w (fp32, uniform in [0.5, 1.5], dv values)."""
    g = torch.Generator(device=device).manual_seed(seed)
    gate = (scale * _normal(tuple(v_shape), g, device)).to(dtype)
    w = 0.5 + torch.rand((v_shape[-1],), generator=g, device=device)
    return gate, w


def make_layer_inputs(B: int, T: int, H: int, dk: int, dv: int, *, dtype=torch.bfloat16, seqlens=None,
                      seed: int = 0, device="cpu", dt_range=(1e-3, 1e-1)) -> dict:
    """Inputs of the operator with the layer's producer steps: raw q, k
    (normal, not normalised; each row scaled by U(0.5, 2)), v, the decay
    gate's projection output f ~ N(0, 1) (dtype), per-head A_log = log A with
    A ~ U(1, 16) and per-(head, channel) dt_bias = softplus^-1(dt) with
    log dt ~ U(log dt_range[0], log dt_range[1]) (fp32; the default is
    Mamba's initialisation range, whose fastest channels decay beyond the
    factorised chunk range in most chunks), beta, S0 and cu_seqlens as
    make_inputs."""
    g = torch.Generator(device=device).manual_seed(seed)
    N = len(seqlens) if seqlens is not None else B
    if seqlens is not None and (B != 1 or T != sum(seqlens)):
        raise ValueError("packed inputs need B == 1 and T == sum(seqlens)")
    q = _normal((B, T, H, dk), g, device) * (0.5 + 1.5 * torch.rand((B, T, H, 1), generator=g, device=device))
    k = _normal((B, T, H, dk), g, device) * (0.5 + 1.5 * torch.rand((B, T, H, 1), generator=g, device=device))
    v = _normal((B, T, H, dv), g, device)
    f = _normal((B, T, H, dk), g, device)
    A_log = torch.log(1.0 + 15.0 * torch.rand((H,), generator=g, device=device))
    lo, hi = math.log(dt_range[0]), math.log(dt_range[1])
    dt = torch.exp(lo + (hi - lo) * torch.rand((H, dk), generator=g, device=device))
    dt_bias = dt + torch.log(-torch.expm1(-dt))
    beta = torch.sigmoid(_normal((B, T, H), g, device))
    S0 = 0.1 * _normal((N, H, dk, dv), g, device)
    cu = None
    if seqlens is not None:
        cu = torch.zeros(N + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(seqlens, dtype=torch.int64), 0).to(torch.int32)
        cu = cu.to(device)
    return dict(q=q.to(dtype), k=k.to(dtype), v=v.to(dtype), f=f.to(dtype), A_log=A_log, dt_bias=dt_bias,
                beta=beta.to(dtype), S0=S0, cu_seqlens=cu)


def workload_inputs(w: Workload, device="cpu", seed_offset: int = 0) -> dict:
    """Inputs for a named workload (``workload(name)``)."""
    return make_inputs(w.B, w.T, w.H, w.dk, w.dv, dtype=w.dtype, gate=w.gate, s0=w.s0,
                       seqlens=w.seqlens, seed=w.seed + seed_offset, device=device)


def decode_step_inputs(N: int, H: int, dk: int, dv: int, step: int, *, dtype=torch.bfloat16,
                       gate: str = "wide", seed: int = BASE_SEED + 4, device="cpu") -> dict:
    """Fresh per-step decode inputs: q, k, log_alpha [N,H,dk]; v [N,H,dv]; beta [N,H]."""
    x = make_inputs(N, 1, H, dk, dv, dtype=dtype, gate=gate, s0="none",
                    seed=seed * 1000003 + step, device=device)
    return {kk: x[kk][:, 0] for kk in ("q", "k", "v", "log_alpha", "beta")}


def decode_state(N: int, H: int, dk: int, dv: int, *, seed: int = BASE_SEED + 4, device="cpu"):
    """Initial decode state ~ N(0, 0.01) (std 0.1), fp32 [N, H, dk, dv]."""
    g = torch.Generator(device=device).manual_seed(seed)
    return 0.1 * _normal((N, H, dk, dv), g, device)
