"""GPU parity of the operator with the Kimi Linear layer's producer steps
fused (kda_chunk_fwd_layer): raw q and k are L2-normalised and the decay gate
log alpha = -exp(A_log) * softplus(f + dt_bias) is computed inside the
tensor-core prefill ("Kimi Linear" summary, section "Configuração do modelo
Kimi Linear"), optionally with the output epilogue.  The oracle composes its
own l2norm, decay_gate, forward and output_gate in fp64.

Tolerance: the bf16 bound, 2e-2 relative L2 per (sequence, head) slice and
per 64-token window of o, and per (sequence, head) slice of S_T.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_110_b200 as kda
import oracle
from gated_delta_rule_110_b200 import inputs as gen
from tests.conftest import max_rel_l2_per_slice, max_rel_l2_per_window

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _bounds(o, cu):
    if cu is None:
        return [(b, 0, o.shape[1]) for b in range(o.shape[0])]
    c = cu.cpu().numpy()
    return [(0, int(c[n]), int(c[n + 1])) for n in range(len(c) - 1)]


def _check(x, o, S, gate=None, w=None, eps=1e-5):
    cu = None if x["cu_seqlens"] is None else x["cu_seqlens"].cpu().numpy()
    y_ref, S_ref = oracle.forward_layer(x["q"], x["k"], x["v"], x["f"], x["A_log"], x["dt_bias"], x["beta"], x["S0"],
                                        cu_seqlens=cu, qk_eps=1e-6, out_gate=gate, norm_weight=w, eps=eps)
    y = o.float().cpu().numpy()
    assert np.all(np.isfinite(y))
    err, err_w = 0.0, 0.0
    for b, a, e in _bounds(y, x["cu_seqlens"]):
        if e > a:
            err = max(err, max_rel_l2_per_slice(y[b, a:e], y_ref[b, a:e], slice_axes=(1,)))
            err_w = max(err_w, max_rel_l2_per_window(y[b, a:e], y_ref[b, a:e]))
    err_S = max_rel_l2_per_slice(S.cpu().numpy(), S_ref, slice_axes=(0, 1))
    assert err <= TOL, f"o rel-L2 {err:.3e} > {TOL}"
    assert err_w <= TOL, f"o rel-L2 on a 64-token window {err_w:.3e} > {TOL}"
    assert err_S <= TOL, f"S_T rel-L2 {err_S:.3e} > {TOL}"


def _run(x, **kw):
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    if kw.get("out_gate") is not None:
        kw["out_gate"] = kw["out_gate"].cuda()
        kw["norm_weight"] = kw["norm_weight"].cuda()
    o, S = kda.kda_chunk_fwd_layer(d["q"], d["k"], d["v"], d["f"], d["A_log"], d["dt_bias"], d["beta"], d["S0"],
                                   d["cu_seqlens"], **kw)
    assert kda.kda_check_device_error() == 0
    return o, S


def test_layer_batched_ragged_tail():
    x = gen.make_layer_inputs(2, 200, 3, 128, 128, seed=61)
    o, S = _run(x)
    _check(x, o, S)


@pytest.mark.parametrize("mode", ["fused", "separate"])
def test_layer_varlen_edges_with_epilogue(mode):
    lens = [1, 63, 64, 65, 0, 130, 200, 33]
    x = gen.make_layer_inputs(1, sum(lens), 2, 128, 128, seqlens=lens, seed=62)
    gate, w = gen.output_gate_inputs(x["v"].shape, seed=63)
    o, S = _run(x, out_gate=gate, norm_weight=w, eps=1e-5, gate_mode=mode)
    _check(x, o, S, gate, w, 1e-5)


def test_layer_strong_decay_takes_exact_path():
    """f = +8 with A up to 16: tens of nats per token, far beyond the
    factorised range in every chunk; and a sequence mixing both paths."""
    x = gen.make_layer_inputs(1, 192, 2, 128, 128, seed=64)
    x["f"] = torch.full_like(x["f"], 8.0)
    o, S = _run(x)
    _check(x, o, S)
    y = gen.make_layer_inputs(1, 256, 2, 128, 128, seed=65)
    y["f"][:, 64:128] = 8.0
    o, S = _run(y)
    _check(y, o, S)


def test_layer_zero_and_tiny_rows():
    """Rows of q or k that are zero (normalised to zero by the epsilon) or
    tiny (scale 1e-3: the epsilon inside the root matters)."""
    x = gen.make_layer_inputs(1, 130, 2, 128, 128, seed=66)
    x["q"][:, 5] = 0
    x["k"][:, 9] = 0
    x["q"][:, 20:30] = (x["q"][:, 20:30].float() * 1e-3).to(x["q"].dtype)
    x["k"][:, 40:44] = (x["k"][:, 40:44].float() * 1e-3).to(x["k"].dtype)
    o, S = _run(x)
    _check(x, o, S)


def test_layer_split_choice_is_bit_identical():
    x = gen.make_layer_inputs(3, 300, 2, 128, 128, seed=67)
    o0, S0 = _run(x)
    for sc, gc in [(1, 2), (3, 0), (0, 5)]:
        o1, S1 = _run(x, state_ctas=sc, grid_ctas=gc)
        assert torch.equal(o0, o1) and torch.equal(S0, S1)


def test_layer_prefill_workload_sampled():
    """Prefill sizes (B4 H16 T4096 d128) from raw inputs, with the epilogue;
    oracle on sampled (b, h)."""
    x = gen.make_layer_inputs(4, 4096, 16, 128, 128, seed=68, device="cuda")
    gate, w = gen.output_gate_inputs(x["v"].shape, seed=69, device="cuda")
    o, S = kda.kda_chunk_fwd_layer(x["q"], x["k"], x["v"], x["f"], x["A_log"], x["dt_bias"], x["beta"], x["S0"],
                                   out_gate=gate, norm_weight=w, eps=1e-5)
    assert kda.kda_check_device_error() == 0
    for b, h in [(0, 0), (1, 9), (3, 15)]:
        sub = {k: x[k][b:b + 1, :, h:h + 1].cpu() for k in ("q", "k", "v", "f", "beta")}
        sub["A_log"] = x["A_log"][h:h + 1].cpu()
        sub["dt_bias"] = x["dt_bias"][h:h + 1].cpu()
        sub["S0"] = x["S0"][b:b + 1, h:h + 1].cpu()
        sub["cu_seqlens"] = None
        _check(sub, o[b:b + 1, :, h:h + 1], S[b:b + 1, h:h + 1], gate[b:b + 1, :, h:h + 1].cpu(), w.cpu(), 1e-5)


def test_layer_sharded_single_rank_is_the_plain_call():
    """kda_chunk_fwd_layer_sharded without a process group runs the library's
    call on the whole batch (the multi-rank split is tested on CPU)."""
    from gated_delta_rule_110_b200.shard import kda_chunk_fwd_layer_sharded
    lens = [70, 130, 64]
    x = {k: (v.cuda() if isinstance(v, torch.Tensor) else v)
         for k, v in gen.make_layer_inputs(1, sum(lens), 2, 128, 128, seqlens=lens, seed=70).items()}
    gate, w = gen.output_gate_inputs(x["v"].shape, seed=71, device="cuda")
    o1, S1, _ = kda_chunk_fwd_layer_sharded(x["q"], x["k"], x["v"], x["f"], x["A_log"], x["dt_bias"], x["beta"],
                                            x["S0"], x["cu_seqlens"], out_gate=gate, norm_weight=w)
    o2, S2 = kda.kda_chunk_fwd_layer(x["q"], x["k"], x["v"], x["f"], x["A_log"], x["dt_bias"], x["beta"], x["S0"],
                                     x["cu_seqlens"], out_gate=gate, norm_weight=w)
    assert kda.kda_check_device_error() == 0
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


# ---------------------------------------------------------------- CUDA-core paths and decode
@pytest.mark.parametrize("d,dtype,tol", [(64, torch.float32, 1e-4), (128, torch.float32, 1e-4),
                                         (128, torch.bfloat16, TOL)])
def test_layer_cuda_core_paths(d, dtype, tol):
    """fp32 io, dk = dv = 64, and the bf16 token-by-token recurrence run the
    producer steps in the CUDA-core kernel (fp32 keeps its 1e-4 bound)."""
    lens = [5, 64, 77]
    x = gen.make_layer_inputs(1, sum(lens), 2, d, d, dtype=dtype, seqlens=lens, seed=72)
    o, S = _run(x, recurrent=(dtype == torch.bfloat16))
    cu = x["cu_seqlens"].numpy()
    o_ref, S_ref = oracle.forward_layer(x["q"], x["k"], x["v"], x["f"], x["A_log"], x["dt_bias"], x["beta"], x["S0"],
                                        cu_seqlens=cu, qk_eps=1e-6)
    y = o.float().cpu().numpy()
    c = [int(v) for v in cu]
    err = max(max_rel_l2_per_slice(y[0, c[n]:c[n + 1]], o_ref[0, c[n]:c[n + 1]], slice_axes=(1,))
              for n in range(len(lens)))
    assert err <= tol
    assert max_rel_l2_per_slice(S.cpu().numpy(), S_ref, slice_axes=(0, 1)) <= tol


def _decode_ref(xs, S, gate=None, w=None, eps=1e-5):
    q, k = oracle.l2norm(xs["q"], 1e-6), oracle.l2norm(xs["k"], 1e-6)
    la = oracle.decay_gate(xs["f"], xs["A_log"], xs["dt_bias"])
    o, S1 = oracle.decode(q, k, xs["v"], la, xs["beta"], S)
    if gate is not None:
        o = oracle.output_gate(o, gate, w, eps)
    return o, S1


@pytest.mark.parametrize("d,dtype,tol", [(128, torch.bfloat16, TOL), (64, torch.float32, 1e-4)])
@pytest.mark.parametrize("epilogue", [False, True])
def test_decode_layer_dense_steps(d, dtype, tol, epilogue):
    N, H = 6, 3
    S = gen.decode_state(N, H, d, d, seed=81).cuda()
    S_ref = S.cpu().double().numpy()
    for step in range(3):
        x = gen.make_layer_inputs(N, 1, H, d, d, dtype=dtype, seed=82 + step)
        xs = {kk: x[kk][:, 0] for kk in ("q", "k", "v", "f", "beta")}
        xs["A_log"], xs["dt_bias"] = x["A_log"], x["dt_bias"]
        gate, w = gen.output_gate_inputs((N, H, d), dtype=dtype, seed=90 + step) if epilogue else (None, None)
        o = kda.kda_decode_step_layer(xs["q"].cuda(), xs["k"].cuda(), xs["v"].cuda(), xs["f"].cuda(),
                                      xs["A_log"].cuda(), xs["dt_bias"].cuda(), xs["beta"].cuda(), S,
                                      out_gate=None if gate is None else gate.cuda(),
                                      norm_weight=None if w is None else w.cuda())
        assert kda.kda_check_device_error() == 0
        o_ref, S_ref = _decode_ref(xs, S_ref, gate, w)
        assert max_rel_l2_per_slice(o.float().cpu().numpy(), o_ref, slice_axes=(0, 1)) <= tol
        assert max_rel_l2_per_slice(S.cpu().numpy(), S_ref, slice_axes=(0, 1)) <= tol


def test_decode_layer_slots_equal_dense():
    """Through pool slots (permuted, one padding entry) the step matches the
    dense call on the gathered rows, bit for bit."""
    N, H, d = 5, 2, 128
    pool = gen.decode_state(8, H, d, d, seed=91).cuda()
    slots = torch.tensor([6, 1, -1, 3, 0], dtype=torch.int32, device="cuda")
    x = gen.make_layer_inputs(N, 1, H, d, d, seed=92, device="cuda")
    args = [x[kk][:, 0] for kk in ("q", "k", "v", "f")] + [x["A_log"], x["dt_bias"], x["beta"][:, 0]]
    dense = torch.zeros((N, H, d, d), device="cuda")
    live = [0, 1, 3, 4]
    dense[live] = pool[slots[live].long()]
    o_d = kda.kda_decode_step_layer(*args, dense)
    pool2 = pool.clone()
    o_s = kda.kda_decode_step_layer(*args, pool2, state_slots=slots)
    assert kda.kda_check_device_error() == 0
    assert torch.equal(o_s[live], o_d[live])
    assert torch.equal(pool2[slots[live].long()], dense[live])
    untouched = [i for i in range(8) if i not in (6, 1, 3, 0)]
    assert torch.equal(pool2[untouched], pool[untouched])
