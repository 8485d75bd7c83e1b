"""Sharding of a prefill across ranks: the partition and the reassembly.

Runs on CPU: two gloo ranks, each computing its shard with the fp64 oracle
(injected as the shard function), gather the outputs; the gathered (o, S_T)
must equal the oracle run on the whole batch, bit for bit (the oracle runs
each (sequence, head) chain on its own, so sharding changes no arithmetic).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from gated_delta_rule_110_b200 import inputs as gen
from gated_delta_rule_110_b200.shard import plan_shards


def _oracle_fwd(q, k, v, la, beta, S0, cu):
    import oracle
    o, S = oracle.forward(q, k, v, la, beta, S0, cu_seqlens=None if cu is None else cu.numpy())
    return torch.from_numpy(o), torch.from_numpy(S)


# ---------------------------------------------------------------- the partition
@pytest.mark.parametrize("lengths,H,world", [
    ([512, 8000, 700, 3000, 1, 0, 4096, 2048], 32, 2),
    ([512, 8000, 700, 3000, 1, 0, 4096, 2048], 32, 8),
    ([4096] * 4, 16, 8),
    ([131072], 32, 8),
    ([10, 20], 3, 2),
    ([5], 1, 4),
])
def test_plan_covers_every_chain_once(lengths, H, world):
    plans = plan_shards(lengths, H, world)
    assert len(plans) == world
    seen = np.zeros((len(lengths), H), dtype=int)
    for p in plans:
        assert 0 <= p.n0 <= p.n1 <= len(lengths) and 0 <= p.h0 <= p.h1 <= H
        seen[p.n0:p.n1, p.h0:p.h1] += 1
    assert (seen == 1).all()
    kinds = {p.kind for p in plans}
    assert len(kinds) == 1
    if kinds == {"seq"}:
        # contiguous, in order
        assert [p.n0 for p in plans[1:]] == [p.n1 for p in plans[:-1]]


def test_plan_balances_tokens():
    lengths = [int(x) for x in np.random.default_rng(1).integers(512, 8193, size=64)]
    plans = plan_shards(lengths, 32, 4)
    loads = [sum(lengths[p.n0:p.n1]) for p in plans]
    assert max(loads) - min(loads) <= max(lengths)


def test_few_sequences_shard_by_head():
    plans = plan_shards([131072], 32, 8)
    assert all(p.kind == "head" for p in plans)
    assert [p.h1 - p.h0 for p in plans] == [4] * 8


# ---------------------------------------------------------------- two gloo ranks
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(name):
    if name == "packed":
        lens = [70, 0, 130, 1, 64, 200]
        return gen.make_inputs(1, sum(lens), 2, 64, 64, dtype=torch.float32, seqlens=lens, seed=61)
    if name == "dense":
        return gen.make_inputs(3, 100, 2, 64, 64, dtype=torch.float32, seed=62)
    if name == "heads":
        return gen.make_inputs(1, 150, 4, 64, 64, dtype=torch.float32, seqlens=[150], seed=63)
    raise KeyError(name)


def _rank_main(rank, world, port, name, out_dir):
    import torch.distributed as dist
    from gated_delta_rule_110_b200.shard import kda_chunk_fwd_sharded
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        x = _case(name)
        o, S, plan = kda_chunk_fwd_sharded(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"],
                                           x["cu_seqlens"], fwd=_oracle_fwd)
        torch.save({"o": o, "S": S, "kind": plan.kind}, os.path.join(out_dir, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,kind", [("packed", "seq"), ("dense", "seq"), ("heads", "head")])
def test_two_gloo_ranks_gather_the_unsharded_result(tmp_path, name, kind):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), name, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    x = _case(name)
    o_ref, S_ref = _oracle_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], x["cu_seqlens"])
    for r in range(world):
        got = torch.load(tmp_path / f"r{r}.pt")
        assert got["kind"] == kind
        assert torch.equal(got["o"], o_ref), f"rank {r}: o differs"
        assert torch.equal(got["S"], S_ref), f"rank {r}: S_T differs"


# ---------------------------------------------------------------- the layer path
def _oracle_layer_fwd(q, k, v, f, beta, S0, cu, gate, A_log, dt_bias, norm_weight=None, eps=1e-5):
    import oracle
    o, S = oracle.forward_layer(q, k, v, f, A_log, dt_bias, beta, S0, cu_seqlens=None if cu is None else cu.numpy(),
                                out_gate=gate, norm_weight=norm_weight, eps=eps)
    return torch.from_numpy(o), torch.from_numpy(S)


def _layer_case(name):
    if name == "packed":
        lens = [70, 0, 130, 1, 64, 200]
        x = gen.make_layer_inputs(1, sum(lens), 2, 32, 32, dtype=torch.float32, seqlens=lens, seed=71)
    else:
        x = gen.make_layer_inputs(1, 150, 4, 32, 32, dtype=torch.float32, seqlens=[150], seed=72)
    gate, w = gen.output_gate_inputs(x["v"].shape, dtype=torch.float32, seed=73)
    return x, gate, w


def _layer_rank_main(rank, world, port, name, out_dir):
    import torch.distributed as dist
    from gated_delta_rule_110_b200.shard import kda_chunk_fwd_layer_sharded
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        x, gate, w = _layer_case(name)
        o, S, plan = kda_chunk_fwd_layer_sharded(x["q"], x["k"], x["v"], x["f"], x["A_log"], x["dt_bias"], x["beta"],
                                                 x["S0"], x["cu_seqlens"], out_gate=gate, norm_weight=w, eps=1e-5,
                                                 fwd=_oracle_layer_fwd)
        torch.save({"o": o, "S": S, "kind": plan.kind}, os.path.join(out_dir, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,kind", [("packed", "seq"), ("heads", "head")])
def test_two_gloo_ranks_layer_path(tmp_path, name, kind):
    """The layer path's extra inputs shard with the rest: the gate projection
    and the output gate with the tokens, A_log and dt_bias with the heads."""
    world = 2
    mp.start_processes(_layer_rank_main, args=(world, _free_port(), name, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    x, gate, w = _layer_case(name)
    o_ref, S_ref = _oracle_layer_fwd(x["q"], x["k"], x["v"], x["f"], x["beta"], x["S0"], x["cu_seqlens"], gate,
                                     x["A_log"], x["dt_bias"], norm_weight=w, eps=1e-5)
    for r in range(world):
        got = torch.load(tmp_path / f"r{r}.pt")
        assert got["kind"] == kind
        assert torch.equal(got["o"], o_ref), f"rank {r}: o differs"
        assert torch.equal(got["S"], S_ref), f"rank {r}: S_T differs"


def _oracle_gated_fwd(q, k, v, la, beta, S0, cu, gate, norm_weight=None, eps=1e-5):
    import oracle
    o, S = oracle.forward(q, k, v, la, beta, S0, cu_seqlens=None if cu is None else cu.numpy())
    return torch.from_numpy(oracle.output_gate(o, gate, norm_weight, eps)), torch.from_numpy(S)


def _gated_rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    from gated_delta_rule_110_b200.shard import kda_chunk_fwd_gated_sharded
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        x = _case("packed")
        gate, w = gen.output_gate_inputs(x["v"].shape, dtype=torch.float32, seed=74)
        o, S, plan = kda_chunk_fwd_gated_sharded(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], gate, w, x["S0"],
                                                 x["cu_seqlens"], fwd=_oracle_gated_fwd)
        torch.save({"o": o, "S": S}, os.path.join(out_dir, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_gated_path(tmp_path):
    world = 2
    mp.start_processes(_gated_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    x = _case("packed")
    gate, w = gen.output_gate_inputs(x["v"].shape, dtype=torch.float32, seed=74)
    o_ref, S_ref = _oracle_gated_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], x["cu_seqlens"],
                                     gate, norm_weight=w)
    for r in range(world):
        got = torch.load(tmp_path / f"r{r}.pt")
        assert torch.equal(got["o"], o_ref) and torch.equal(got["S"], S_ref)
