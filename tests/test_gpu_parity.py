"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerance (stated with the workloads): the largest relative L2 error over
(sequence, head) slices, ||x - x_oracle|| / ||x_oracle||, must be <= 1e-4 for
fp32 inputs and <= 2e-2 for bf16 inputs with the fp32 state.  o slices are
[tokens, dv]; S_T slices are [dk, dv].  Both sides read the same input bits
(the oracle upcasts the bf16 / fp32 tensors the kernels consumed).
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_110_b200 as kda
import oracle
from gated_delta_rule_110_b200 import inputs as gen
from tests.conftest import max_rel_l2_per_slice, max_rel_l2_per_window

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
TOL_F32 = 1e-4


def _dev(x):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def _oracle_fwd(x):
    cu = None if x["cu_seqlens"] is None else x["cu_seqlens"].cpu().numpy()
    return oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], cu_seqlens=cu)


def _check_fwd(x, tol, o=None, S=None, seq_slices=None):
    """Compare kernel output (o, S) with the oracle.

    Two measures, both at ``tol``: the per-(sequence, head) relative L2 error
    of the stated tolerance, and the same error on every 64-token window of
    each sequence (aligned to the sequence start, i.e. to its chunks), so a
    mistake confined to one chunk cannot hide in a long sequence's norm.
    """
    o_ref, S_ref = _oracle_fwd(x)
    o = o.float().cpu().numpy()
    S = S.cpu().numpy()
    cu = x["cu_seqlens"]
    if cu is None:
        T = o.shape[1]
        bounds = [(b, 0, T) for b in range(o.shape[0])]
    else:
        c = cu.cpu().numpy()
        bounds = [(0, int(c[n]), int(c[n + 1])) for n in range(len(c) - 1)]
    err_o, err_w = 0.0, 0.0
    for b, a, e in bounds:
        if e > a:
            err_o = max(err_o, max_rel_l2_per_slice(o[b, a:e], o_ref[b, a:e], slice_axes=(1,)))
            err_w = max(err_w, max_rel_l2_per_window(o[b, a:e], o_ref[b, a:e]))
    err_S = max_rel_l2_per_slice(S, S_ref, slice_axes=(0, 1))
    assert err_o <= tol, f"o rel-L2 {err_o:.3e} > {tol}"
    assert err_w <= tol, f"o rel-L2 on a 64-token window {err_w:.3e} > {tol}"
    assert err_S <= tol, f"S_T rel-L2 {err_S:.3e} > {tol}"
    return err_o, err_S


def _run(x, **kw):
    xd = _dev(x)
    o, S = kda.kda_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["S0"],
                             xd["cu_seqlens"], **kw)
    assert kda.kda_check_device_error() == 0
    return o, S


# ---------------------------------------------------------------- decode
@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.float32), (128, torch.float32)])
def test_decode_step_matches_oracle(d, dtype):
    N, H = 24, 4
    S = gen.decode_state(N, H, d, d, seed=5).cuda()
    S_ref = S.cpu().double().numpy()
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    for step in range(3):
        x = _dev(gen.decode_step_inputs(N, H, d, d, step, dtype=dtype, seed=77))
        o = kda.kda_decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S)
        o_ref, S_ref = oracle.decode(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S_ref)
        eo = max_rel_l2_per_slice(o.float().cpu().numpy(), o_ref, slice_axes=(0, 1))
        eS = max_rel_l2_per_slice(S.cpu().numpy(), S_ref, slice_axes=(0, 1))
        assert eo <= tol and eS <= tol, (step, eo, eS)


def test_decode_full_size_sampled():
    """Decode workload sizes (256 sequences x 32 heads, d=128, bf16); sampled slices."""
    w = gen.workload("decode")
    N, H, d = w.B, w.H, w.dk
    S = gen.decode_state(N, H, d, d, device="cuda")
    S_host = S.cpu().double().numpy()
    idx = np.random.default_rng(0).choice(N * H, size=64, replace=False)
    for step in range(2):
        x = gen.decode_step_inputs(N, H, d, d, step, device="cuda")
        o = kda.kda_decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S)
        n_i, h_i = idx // H, idx % H
        sub = {k: v.cpu()[n_i, h_i][:, None] for k, v in x.items()}
        o_ref, S_new = oracle.decode(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"],
                                     S_host[n_i, h_i][:, None])
        S_host[n_i, h_i] = S_new[:, 0]
        eo = max_rel_l2_per_slice(o.float().cpu().numpy()[n_i, h_i], o_ref[:, 0], slice_axes=(0,))
        eS = max_rel_l2_per_slice(S.cpu().numpy()[n_i, h_i], S_host[n_i, h_i], slice_axes=(0,))
        assert eo <= TOL_BF16 and eS <= TOL_BF16, (step, eo, eS)


# ---------------------------------------------------------------- fp32 path
def test_oracle_workload_fp32():
    """The oracle-scale workload (B1 H2 T256 d64 C64, fp32) at 1e-4."""
    x = gen.workload_inputs(gen.workload("oracle"))
    o, S = _run(x)
    _check_fwd(x, TOL_F32, o, S)


@pytest.mark.parametrize("d", [64, 128])
def test_fp32_ragged_varlen(d):
    x = gen.make_inputs(1, 1 + 63 + 130 + 7, 3, d, d, dtype=torch.float32, seqlens=[1, 63, 0, 130, 7],
                        seed=3)
    o, S = _run(x)
    _check_fwd(x, TOL_F32, o, S)


# ---------------------------------------------------------------- tensor-core path
def test_tc_small_batched_ragged_tail():
    """B=2, T=200 (three full chunks and a ragged tail), H=3, d=128, bf16."""
    x = gen.make_inputs(2, 200, 3, 128, 128, seed=11)
    o, S = _run(x)
    _check_fwd(x, TOL_BF16, o, S)


def test_tc_varlen_edges():
    """Sequences of length 1, 63, 64, 65, 0, 130 and 200 packed together."""
    lens = [1, 63, 64, 65, 0, 130, 200]
    x = gen.make_inputs(1, sum(lens), 2, 128, 128, seqlens=lens, seed=12)
    o, S = _run(x)
    _check_fwd(x, TOL_BF16, o, S)


def test_tc_fp32_gates():
    x = gen.make_inputs(1, 192, 2, 128, 128, gate_dtype=torch.float32, seed=13)
    o, S = _run(x)
    _check_fwd(x, TOL_BF16, o, S)


def test_tc_no_initial_state():
    x = gen.make_inputs(2, 130, 2, 128, 128, s0="none", seed=14)
    o, S = _run(x)
    x["S0"] = None
    _check_fwd(x, TOL_BF16, o, S)


def test_tc_zero_state_short_sequences():
    """Sequences of 1-3 tokens from a zero state: the output of a token is
    beta (q . k) v plus few other terms, so a nearly orthogonal q, k pair
    makes each (sequence, head) slice ill-conditioned.  The diagonal of the
    intra-chunk product must not lose q . k to the rounding of the scaled
    bf16 operands."""
    lens = [1] * 24 + [2] * 8 + [3] * 8
    x = gen.make_inputs(1, sum(lens), 4, 128, 128, seqlens=lens, s0="none", seed=33)
    o, S = _run(x)
    _check_fwd(x, TOL_BF16, o, S)


def test_tc_strong_decay_takes_exact_path():
    """log_alpha = -5 everywhere: each chunk decays 320 nats, beyond the
    factorised form's range; the exact path must still match."""
    x = gen.make_inputs(1, 160, 2, 128, 128, seed=15)
    x["log_alpha"] = torch.full_like(x["log_alpha"], -5.0)
    o, S = _run(x)
    _check_fwd(x, TOL_BF16, o, S)


def test_tc_no_decay():
    x = gen.make_inputs(1, 192, 2, 128, 128, gate="zero", seed=16)
    o, S = _run(x)
    _check_fwd(x, TOL_BF16, o, S)


def test_tc_mixed_fast_and_exact_chunks():
    """Half the chunks decay beyond the fast path's span, half do not."""
    x = gen.make_inputs(1, 256, 2, 128, 128, seed=17)
    la = x["log_alpha"].float()
    la[:, 64:128] = -4.0
    la[:, 192:256] = -3.0
    x["log_alpha"] = la.to(torch.bfloat16)
    o, S = _run(x)
    _check_fwd(x, TOL_BF16, o, S)


def test_tc_prefill_workload_sampled():
    """Prefill workload at full size (B4 H16 T4096 d128); oracle on sampled (b, h)."""
    w = gen.workload("prefill")
    x = gen.workload_inputs(w, device="cuda")
    o, S = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    assert kda.kda_check_device_error() == 0
    rng = np.random.default_rng(1)
    for b, h in [(0, 0), (3, 15), (int(rng.integers(4)), int(rng.integers(16)))]:
        sub = {k: x[k][b:b + 1, :, h:h + 1].cpu() for k in ("q", "k", "v", "log_alpha")}
        sub["beta"] = x["beta"][b:b + 1, :, h:h + 1].cpu()
        sub["S0"] = x["S0"][b:b + 1, h:h + 1].cpu()
        sub["cu_seqlens"] = None
        _check_fwd(sub, TOL_BF16, o[b:b + 1, :, h:h + 1], S[b:b + 1, h:h + 1])


# ---------------------------------------------------------------- properties
def test_tc_path_matches_cuda_core_path():
    """Same inputs through the tensor-core path and the fp32 token-by-token
    CUDA-core recurrence (KDA_FLAG_PATH_RECURRENT): they agree within bf16
    error."""
    x = _dev(gen.make_inputs(1, 300, 2, 128, 128, seed=21))
    o1, S1 = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    o2, S2 = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], recurrent=True)
    assert max_rel_l2_per_slice(o1.float().cpu(), o2.float().cpu(), (0, 2)) < TOL_BF16
    assert max_rel_l2_per_slice(S1.cpu(), S2.cpu(), (0, 1)) < TOL_BF16


@pytest.mark.parametrize("lens", [[1, 63, 64, 65, 0, 130, 200], [300]])
def test_recurrent_path_bf16_matches_oracle(lens):
    x = gen.make_inputs(1, sum(lens), 2, 128, 128, seqlens=lens, seed=27)
    o, S = _run(x, recurrent=True)
    _check_fwd(x, TOL_BF16, o, S)


def test_tc_split_resume():
    x = _dev(gen.make_inputs(1, 320, 2, 128, 128, seed=22))
    o, S = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    T1 = 128
    sl = lambda t, a, b: t[:, a:b].contiguous()
    oa, Sa = kda.kda_chunk_fwd(*(sl(x[k], 0, T1) for k in ("q", "k", "v", "log_alpha", "beta")), x["S0"])
    ob, Sb = kda.kda_chunk_fwd(*(sl(x[k], T1, 320) for k in ("q", "k", "v", "log_alpha", "beta")), Sa)
    assert max_rel_l2_per_slice(torch.cat([oa, ob], 1).float().cpu(), o.float().cpu(), (0, 2)) < 1e-2
    assert max_rel_l2_per_slice(Sb.cpu(), S.cpu(), (0, 1)) < 1e-2


def test_decode_steps_equal_prefill():
    T, N, H, d = 40, 3, 2, 128
    x = _dev(gen.make_inputs(N, T, H, d, d, seed=23))
    o, S = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    Sd = x["S0"].clone()
    outs = []
    for t in range(T):
        outs.append(kda.kda_decode_step(*(x[k][:, t].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")),
                                        Sd))
    od = torch.stack(outs, 1)
    assert max_rel_l2_per_slice(od.float().cpu(), o.float().cpu(), (0, 2)) < TOL_BF16
    assert max_rel_l2_per_slice(Sd.cpu(), S.cpu(), (0, 1)) < TOL_BF16


def test_tc_varlen_equals_separate_calls():
    lens = [70, 5, 129]
    x = _dev(gen.make_inputs(1, sum(lens), 2, 128, 128, seqlens=lens, seed=24))
    o, S = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], x["cu_seqlens"])
    c = [0, 70, 75, 204]
    for n in range(3):
        a, b = c[n], c[n + 1]
        on, Sn = kda.kda_chunk_fwd(*(x[k][:, a:b].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")),
                                   x["S0"][n:n + 1].contiguous())
        # identical arithmetic per sequence: bit-identical results
        assert torch.equal(on, o[:, a:b]) and torch.equal(Sn, S[n:n + 1])


def test_tc_deterministic():
    x = _dev(gen.make_inputs(2, 257, 2, 128, 128, seed=25))
    r1 = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    for _ in range(3):
        r2 = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
        assert torch.equal(r1[0], r2[0]) and torch.equal(r1[1], r2[1])


def test_final_state_may_alias_initial_state():
    x = _dev(gen.make_inputs(1, 100, 2, 128, 128, seed=26))
    o, S = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    S_io = x["S0"].clone()
    o2, _ = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S_io, S_T=S_io)
    assert torch.equal(o, o2) and torch.equal(S, S_io)


# ---------------------------------------------------------------- pipelined-path scheduling
@pytest.mark.parametrize("state_ctas,grid_ctas", [(1, 2), (1, 0), (2, 3), (3, 0), (0, 4), (0, 0)])
def test_tc_state_cta_splits(state_ctas, grid_ctas):
    """Packed sequences (one empty, ragged tails) over 3 heads, with the CTA
    split forced: one state CTA walking every chain, a single transform CTA
    feeding it, uneven streams.  Results must not depend on the split."""
    lens = [130, 0, 64, 1, 257, 70]
    x = gen.make_inputs(1, sum(lens), 3, 128, 128, seqlens=lens, seed=31)
    xd = _dev(x)
    o, S = kda.kda_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["S0"], xd["cu_seqlens"],
                             state_ctas=state_ctas, grid_ctas=grid_ctas)
    assert kda.kda_check_device_error() == 0
    _check_fwd(x, TOL_BF16, o, S)


def test_tc_split_choice_is_bit_identical():
    """Every chunk is computed by the same arithmetic whichever CTA runs it."""
    lens = [200, 77, 128]
    xd = _dev(gen.make_inputs(1, sum(lens), 4, 128, 128, seqlens=lens, seed=32))
    args = (xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["S0"], xd["cu_seqlens"])
    ref = kda.kda_chunk_fwd(*args)
    for sc, gc in ((1, 2), (2, 0), (5, 7)):
        o, S = kda.kda_chunk_fwd(*args, state_ctas=sc, grid_ctas=gc)
        assert torch.equal(o, ref[0]) and torch.equal(S, ref[1]), (sc, gc)
