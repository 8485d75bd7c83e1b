"""GPU parity of the output epilogue (kda_chunk_fwd_gated): the prefill
followed by the per-head RMSNorm and the sigmoid output gate of the Kimi
Linear model ("Kimi Linear" summary, section on the model configuration),
either fused into the tensor-core kernel's output warps or as a separate pass
over o.  The oracle runs its token-by-token forward and then its own
output_gate on the fp64 result.

Tolerance: the bf16 bound of the ungated path, 2e-2 relative L2 per
(sequence, head) slice and per 64-token window.  The normalisation divides
each token by its own root mean square, so the gated error is the per-token
relative error of o, at most that of the ungated output on the same tokens
for the well-conditioned random inputs used here.
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


def _dev(x):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def _bounds(o, cu):
    if cu is None:
        return [(b, 0, o.shape[1]) for b in range(o.shape[0])]
    c = cu.cpu().numpy()
    return [(0, int(c[n]), int(c[n + 1])) for n in range(len(c) - 1)]


def _check(x, gate, w, eps, o, S, tol=TOL):
    cu = None if x["cu_seqlens"] is None else x["cu_seqlens"].cpu().numpy()
    o_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], cu_seqlens=cu)
    y_ref = oracle.output_gate(o_ref, gate, w, eps)
    y = o.float().cpu().numpy()
    assert np.all(np.isfinite(y))
    err, err_w = 0.0, 0.0
    for b, a, e in _bounds(y, x["cu_seqlens"]):
        if e > a:
            err = max(err, max_rel_l2_per_slice(y[b, a:e], y_ref[b, a:e], slice_axes=(1,)))
            err_w = max(err_w, max_rel_l2_per_window(y[b, a:e], y_ref[b, a:e]))
    err_S = max_rel_l2_per_slice(S.cpu().numpy(), S_ref, slice_axes=(0, 1))
    assert err <= tol, f"gated o rel-L2 {err:.3e} > {tol}"
    assert err_w <= tol, f"gated o rel-L2 on a 64-token window {err_w:.3e} > {tol}"
    assert err_S <= tol, f"S_T rel-L2 {err_S:.3e} > {tol}"
    return err


def _run(x, gate, w, eps, **kw):
    xd = _dev(x)
    o, S = kda.kda_chunk_fwd_gated(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], gate.cuda(), w.cuda(),
                                   xd["S0"], xd["cu_seqlens"], eps=eps, **kw)
    assert kda.kda_check_device_error() == 0
    return o, S


MODES = ["fused", "separate"]


@pytest.mark.parametrize("mode", MODES)
def test_gated_batched_ragged_tail(mode):
    """B=2, T=200 (three full chunks, a 8-token tail), H=3: full 32-row
    tiles go out by tensor store, the tail row by row."""
    x = gen.make_inputs(2, 200, 3, 128, 128, seed=41)
    gate, w = gen.output_gate_inputs(x["v"].shape, seed=42)
    o, S = _run(x, gate, w, 1e-5, gate_mode=mode)
    _check(x, gate, w, 1e-5, o, S)


@pytest.mark.parametrize("mode", MODES)
def test_gated_varlen_edges(mode):
    lens = [1, 63, 64, 65, 0, 130, 200, 31, 33]
    x = gen.make_inputs(1, sum(lens), 2, 128, 128, seqlens=lens, seed=43)
    gate, w = gen.output_gate_inputs(x["v"].shape, seed=44)
    o, S = _run(x, gate, w, 1e-6, gate_mode=mode)
    _check(x, gate, w, 1e-6, o, S)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("scale,eps", [(0.0, 1e-5), (30.0, 1e-5), (1.0, 1.0), (3.0, 0.0)])
def test_gated_gate_and_epsilon_ranges(scale, eps, mode):
    """A gate at 0 (every sigmoid 1/2), saturated gates (|g| up to ~100: the
    sigmoid at 0 or 1), an epsilon comparable to the mean square, and none."""
    x = gen.make_inputs(1, 160, 2, 128, 128, seed=45)
    gate, w = gen.output_gate_inputs(x["v"].shape, scale=scale, seed=46)
    o, S = _run(x, gate, w, eps, gate_mode=mode)
    _check(x, gate, w, eps, o, S)


@pytest.mark.parametrize("d,dtype,tol", [(64, torch.float32, 1e-4), (128, torch.float32, 1e-4),
                                         (128, torch.bfloat16, TOL)])
def test_gated_cuda_core_paths(d, dtype, tol):
    """fp32 io, dk = dv = 64, and the bf16 token-by-token recurrence: the
    CUDA-core kernel applies the epilogue to each token's o (fp32 io with
    the accurate exp, within the fp32 bound)."""
    lens = [5, 64, 77]
    x = gen.make_inputs(1, sum(lens), 2, d, d, dtype=dtype, seqlens=lens, seed=50)
    gate, w = gen.output_gate_inputs(x["v"].shape, dtype=dtype, seed=51)
    o, S = _run(x, gate, w, 1e-5, recurrent=(dtype == torch.bfloat16))
    _check(x, gate, w, 1e-5, o, S, tol)


@pytest.mark.parametrize("mode", MODES)
def test_gated_state_and_split_match_ungated(mode):
    """The epilogue changes o only: S_T is bit-identical to the ungated call's,
    for several state / transform CTA splits."""
    x = _dev(gen.make_inputs(3, 300, 2, 128, 128, seed=47))
    gate, w = gen.output_gate_inputs(x["v"].shape, seed=48, device="cuda")
    _, S_plain = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    outs = []
    for sc, gc in [(0, 0), (1, 2), (3, 0)]:
        o, S = kda.kda_chunk_fwd_gated(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], gate, w, x["S0"],
                                       state_ctas=sc, grid_ctas=gc, gate_mode=mode)
        assert kda.kda_check_device_error() == 0
        assert torch.equal(S, S_plain)
        outs.append(o)
    assert all(torch.equal(outs[0], oo) for oo in outs[1:])


def test_fused_and_separate_agree():
    """The two placements of the epilogue differ only in where o is rounded
    to bf16 (the fused one normalises the fp32 products): they agree to
    within a few bf16 rounding steps everywhere."""
    x = _dev(gen.make_inputs(2, 700, 4, 128, 128, seed=52))
    gate, w = gen.output_gate_inputs(x["v"].shape, seed=53, device="cuda")
    args = (x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], gate, w, x["S0"])
    of, Sf = kda.kda_chunk_fwd_gated(*args, gate_mode="fused")
    os_, Ss = kda.kda_chunk_fwd_gated(*args, gate_mode="separate")
    oa, _ = kda.kda_chunk_fwd_gated(*args)
    assert kda.kda_check_device_error() == 0
    assert torch.equal(Sf, Ss)
    assert torch.equal(oa, of) or torch.equal(oa, os_)
    diff = (of.float() - os_.float()).abs()
    assert float(diff.max()) <= 0.05 * float(of.float().abs().max())
    assert float(diff.norm() / of.float().norm()) <= 5e-3


@pytest.mark.parametrize("mode", ["auto"] + MODES)
def test_gated_prefill_workload_sampled(mode):
    """Prefill workload at full size (B4 H16 T4096 d128) with the epilogue;
    oracle on sampled (b, h)."""
    wl = gen.workload("prefill")
    x = gen.workload_inputs(wl, device="cuda")
    gate, w = gen.output_gate_inputs(x["v"].shape, seed=49, device="cuda")
    o, S = kda.kda_chunk_fwd_gated(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], gate, w, x["S0"], eps=1e-5,
                                   gate_mode=mode)
    assert kda.kda_check_device_error() == 0
    for b, h in [(0, 0), (2, 7), (3, 15)]:
        sub = {k: x[k][b:b + 1, :, h:h + 1].cpu() for k in ("q", "k", "v", "log_alpha", "beta")}
        sub["S0"] = x["S0"][b:b + 1, h:h + 1].cpu()
        sub["cu_seqlens"] = None
        _check(sub, gate[b:b + 1, :, h:h + 1].cpu(), w.cpu(), 1e-5, o[b:b + 1, :, h:h + 1], S[b:b + 1, h:h + 1])
