"""Data-parallel sharding of a prefill across ranks (one process per GPU).

The (sequence, head) chains of the recurrence are independent: the chunkwise
form ("Algoritmo paralelo por chunks" on the Kimi Linear summary page) only
carries the state from one chunk of a sequence to the next chunk of the same
sequence and head.  So a batch shards across ranks with no exchange inside
the path: each rank runs kda_chunk_fwd on its own sequences (or heads) and
the outputs are gathered once at the end, if the caller wants them on every
rank at all.

Two partitions, both zero-copy for their inputs where the layout allows:

* by sequence (``plan.kind == "seq"``): rank r owns a contiguous run of
  sequences, chosen to balance token counts.  In the packed layout that run
  is a contiguous block of token rows, so the inputs are views.
* by head (``plan.kind == "head"``): when there are fewer sequences than
  ranks (a single long prompt), rank r owns a contiguous block of heads; the
  head-sliced inputs are strided and are copied once.

Collectives go through ``torch.distributed`` (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class ShardPlan:
    """What one rank computes: sequences [n0, n1) of all heads (kind "seq"),
    or heads [h0, h1) of all sequences (kind "head")."""
    kind: str
    n0: int
    n1: int
    h0: int
    h1: int


def _seq_bounds(lengths, world_size):
    """Split sequences into world_size contiguous runs with balanced token
    counts (greedy on the running total; empty runs allowed)."""
    total = sum(lengths)
    bounds = [0]
    acc = 0
    n = 0
    for r in range(1, world_size):
        target = total * r / world_size
        while n < len(lengths) and acc + lengths[n] / 2 <= target:
            acc += lengths[n]
            n += 1
        bounds.append(max(n, bounds[-1]))
    bounds.append(len(lengths))
    return bounds


def plan_shards(lengths, H: int, world_size: int):
    """One ShardPlan per rank for sequences of the given lengths and H heads."""
    if world_size < 1:
        raise ValueError("world_size must be >= 1")
    N = len(lengths)
    if N >= world_size or H < world_size:
        b = _seq_bounds(list(lengths), world_size)
        return [ShardPlan("seq", b[r], b[r + 1], 0, H) for r in range(world_size)]
    hb = [(H * r) // world_size for r in range(world_size + 1)]
    return [ShardPlan("head", 0, N, hb[r], hb[r + 1]) for r in range(world_size)]


def _lengths(q, cu_seqlens):
    if cu_seqlens is None:
        B, T = q.shape[0], q.shape[1]
        return [T] * B
    c = [int(x) for x in cu_seqlens.tolist()]
    return [c[i + 1] - c[i] for i in range(len(c) - 1)]


def local_inputs(plan: ShardPlan, q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, token_extras=(),
                 head_extras=()):
    """This rank's slice of the inputs, in the library's layouts.

    Returns (q, k, v, log_alpha, beta, S0, cu_seqlens, *token_extras,
    *head_extras) for the shard; for a sequence shard of a packed batch,
    cu_seqlens is rebased to start at 0.  ``token_extras`` are laid out like
    q ([B, T, H, ...]) and sliced with it; ``head_extras`` have the head
    axis first ([H, ...]) and are sliced only by a head shard."""
    if plan.kind == "seq":
        if cu_seqlens is None:
            sl = slice(plan.n0, plan.n1)
            xs = [t[sl] for t in (q, k, v, log_alpha, beta, *token_extras)]
            return (*xs[:5], None if S0 is None else S0[sl], None, *xs[5:], *head_extras)
        c = cu_seqlens
        a, e = int(c[plan.n0]), int(c[plan.n1])
        xs = [t[:, a:e] for t in (q, k, v, log_alpha, beta, *token_extras)]
        cu = (c[plan.n0:plan.n1 + 1] - c[plan.n0]).contiguous()
        return (*xs[:5], None if S0 is None else S0[plan.n0:plan.n1], cu, *xs[5:], *head_extras)
    hs = slice(plan.h0, plan.h1)
    xs = [t[:, :, hs].contiguous() for t in (q, k, v, log_alpha, beta, *token_extras)]
    hx = [t[hs].contiguous() for t in head_extras]
    return (*xs[:5], None if S0 is None else S0[:, hs].contiguous(), cu_seqlens, *xs[5:], *hx)


def _gather_padded(t, group, dist):
    """all_gather of tensors whose first dimension differs across ranks."""
    import torch
    world = dist.get_world_size(group)
    n = torch.tensor([t.shape[0]], dtype=torch.int64, device=t.device)
    sizes = [torch.zeros_like(n) for _ in range(world)]
    dist.all_gather(sizes, n, group=group)
    m = max(int(s.item()) for s in sizes)
    pad = torch.zeros((m,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    pad[: t.shape[0]] = t
    out = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(out, pad, group=group)
    return [o[: int(s.item())] for o, s in zip(out, sizes)]


def kda_chunk_fwd_sharded(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, *, group=None, fwd=None,
                          gather: bool = True, token_extras=(), head_extras=()):
    """Prefill of a batch split across the ranks of ``group``.

    Every rank passes the same full inputs (or at least the same shapes and
    cu_seqlens; only its own shard is read).  ``fwd`` computes one shard,
    called as fwd(q, k, v, log_alpha, beta, S0, cu_seqlens, *token_extras,
    *head_extras) on the shard's slices (see local_inputs), and defaults to
    the library's kda_chunk_fwd.  With ``gather`` every rank returns the full
    (o, S_T); otherwise its own shard, its plan, and no collective is issued.
    """
    import torch
    import torch.distributed as dist
    if fwd is None:
        from . import kda_chunk_fwd as fwd
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    H = q.shape[2]
    plans = plan_shards(_lengths(q, cu_seqlens), H, world)
    plan = plans[rank]
    loc = local_inputs(plan, q, k, v, log_alpha, beta, S0, cu_seqlens, token_extras, head_extras)
    lq, lv = loc[0], loc[2]
    empty = (plan.n1 - plan.n0) == 0 or (plan.h1 - plan.h0) == 0
    if empty:
        o_loc = lv.new_zeros(lv.shape)
        S_loc = lq.new_zeros((plan.n1 - plan.n0, plan.h1 - plan.h0, q.shape[3], v.shape[3]), dtype=torch.float32)
    else:
        o_loc, S_loc = fwd(*loc)
    if not gather or world == 1:
        return o_loc, S_loc, plan
    # rows of o along the sharded axis first, so that shards concatenate
    if plan.kind == "seq":
        o_rows = o_loc.reshape(-1, *o_loc.shape[2:]) if cu_seqlens is not None else o_loc
        o_parts = _gather_padded(o_rows, group, dist)
        S_parts = _gather_padded(S_loc, group, dist)
        S_T = torch.cat(S_parts, 0)
        if cu_seqlens is not None:
            o = torch.cat(o_parts, 0).reshape(v.shape)
        else:
            o = torch.cat(o_parts, 0)
        return o, S_T, plan
    o_parts = _gather_padded(o_loc.permute(2, 0, 1, 3).contiguous(), group, dist)
    S_parts = _gather_padded(S_loc.permute(1, 0, 2, 3).contiguous(), group, dist)
    o = torch.cat(o_parts, 0).permute(1, 2, 0, 3).contiguous()
    S_T = torch.cat(S_parts, 0).permute(1, 0, 2, 3).contiguous()
    return o, S_T, plan


def kda_chunk_fwd_layer_sharded(q, k, v, gate_f, A_log, dt_bias, beta, S0=None, cu_seqlens=None, *, out_gate=None,
                                norm_weight=None, eps: float = 1e-5, group=None, fwd=None, gather: bool = True):
    """kda_chunk_fwd_layer (raw q, k and the decay gate's projection in; the
    optional output epilogue) split across the ranks of ``group`` as
    kda_chunk_fwd_sharded splits kda_chunk_fwd: gate_f and out_gate are
    sliced like q, A_log and dt_bias by head.  ``fwd`` (default: the
    library's kda_chunk_fwd_layer) is called as fwd(q, k, v, gate_f, beta,
    S0, cu_seqlens, out_gate, A_log, dt_bias, norm_weight=..., eps=...)."""
    if fwd is None:
        from . import kda_chunk_fwd_layer

        def fwd(lq, lk, lv, lf, lb, ls0, lcu, lgate, lA, lbias, norm_weight=None, eps=1e-5):
            return kda_chunk_fwd_layer(lq, lk, lv, lf, lA, lbias, lb, ls0, lcu, out_gate=lgate,
                                       norm_weight=norm_weight, eps=eps)
    tok = (out_gate,) if out_gate is not None else ()

    def shard_fwd(lq, lk, lv, lf, lb, ls0, lcu, *rest):
        lgate = rest[0] if out_gate is not None else None
        lA, lbias = rest[-2], rest[-1]
        return fwd(lq, lk, lv, lf, lb, ls0, lcu, lgate, lA, lbias, norm_weight=norm_weight, eps=eps)
    return kda_chunk_fwd_sharded(q, k, v, gate_f, beta, S0, cu_seqlens, group=group, fwd=shard_fwd, gather=gather,
                                 token_extras=tok, head_extras=(A_log, dt_bias))


def kda_chunk_fwd_gated_sharded(q, k, v, log_alpha, beta, out_gate, norm_weight, S0=None, cu_seqlens=None, *,
                                eps: float = 1e-5, group=None, fwd=None, gather: bool = True):
    """kda_chunk_fwd_gated (prefill, then the per-head RMSNorm and output
    gate) split across the ranks of ``group``: out_gate is sliced like q.
    ``fwd`` (default: the library's kda_chunk_fwd_gated) is called as
    fwd(q, k, v, log_alpha, beta, S0, cu_seqlens, out_gate, norm_weight=...,
    eps=...)."""
    if fwd is None:
        from . import kda_chunk_fwd_gated

        def fwd(lq, lk, lv, la, lb, ls0, lcu, lgate, norm_weight=None, eps=1e-5):
            return kda_chunk_fwd_gated(lq, lk, lv, la, lb, lgate, norm_weight, ls0, lcu, eps=eps)

    def shard_fwd(lq, lk, lv, la, lb, ls0, lcu, lgate):
        return fwd(lq, lk, lv, la, lb, ls0, lcu, lgate, norm_weight=norm_weight, eps=eps)
    return kda_chunk_fwd_sharded(q, k, v, log_alpha, beta, S0, cu_seqlens, group=group, fwd=shard_fwd,
                                 gather=gather, token_extras=(out_gate,))
