"""GPU parity at the full sizes of the benchmark workloads.

Each test runs one workload at its stated size through the C ABI, in the
launch configuration the benchmark times, and checks it against the fp64
oracle on a seeded subset the oracle finishes in seconds:

* varlen  -- 8 packed sequences of U{512..8192} tokens, H=32, d=128, bf16:
  every sequence, a seeded subset of heads; o (per sequence and per 64-token
  window) and S_T.
* long    -- B=1, H=32, T=131072, near-1 per-channel decay: o on the last
  4096 tokens and the full S_T of a seeded 8-head subset.
* decode  -- 256 sequences x 32 heads, 1000 sequential steps updating the
  state in place: o of 64 sampled (sequence, head) pairs at every step and
  their state after the last step.

Tolerance: the largest relative L2 error over (sequence, head) slices must
be <= 2e-2 (bf16 inputs, fp32 state), on o and on S_T.
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


def _host(t, heads):
    return t[:, :, heads].cpu() if t.dim() >= 3 else t


def test_varlen_workload_full_size():
    w = gen.workload("varlen")
    x = gen.workload_inputs(w, device="cuda")
    o, S = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], x["cu_seqlens"])
    assert kda.kda_check_device_error() == 0
    heads = sorted(np.random.default_rng(3).choice(w.H, size=4, replace=False).tolist())
    sub = {k: x[k][:, :, heads].cpu() for k in ("q", "k", "v", "log_alpha", "beta")}
    cu = x["cu_seqlens"].cpu().numpy()
    o_ref, S_ref = oracle.forward(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"],
                                  x["S0"][:, heads].cpu(), cu_seqlens=cu)
    o_h = o[:, :, heads].float().cpu().numpy()
    for n in range(len(cu) - 1):
        a, b = int(cu[n]), int(cu[n + 1])
        e = max_rel_l2_per_slice(o_h[0, a:b], o_ref[0, a:b], slice_axes=(1,))
        ew = max_rel_l2_per_window(o_h[0, a:b], o_ref[0, a:b])
        assert e <= TOL_BF16 and ew <= TOL_BF16, (n, b - a, e, ew)
    eS = max_rel_l2_per_slice(S[:, heads].cpu().numpy(), S_ref, slice_axes=(0, 1))
    assert eS <= TOL_BF16, eS


def test_long_context_workload_full_size():
    w = gen.workload("long")
    x = gen.workload_inputs(w, device="cuda")
    o, S = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    assert kda.kda_check_device_error() == 0
    heads = sorted(np.random.default_rng(4).choice(w.H, size=8, replace=False).tolist())
    sub = {k: x[k][:, :, heads].cpu() for k in ("q", "k", "v", "log_alpha", "beta")}
    o_ref, S_ref = oracle.forward(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"],
                                  x["S0"][:, heads].cpu())
    tail = 4096
    o_t = o[0, -tail:, heads].float().cpu().numpy()
    r_t = o_ref[0, -tail:]
    e = max_rel_l2_per_slice(o_t, r_t, slice_axes=(1,))
    ew = max_rel_l2_per_window(o_t, r_t)
    eS = max_rel_l2_per_slice(S[:, heads].cpu().numpy(), S_ref, slice_axes=(0, 1))
    assert e <= TOL_BF16 and ew <= TOL_BF16 and eS <= TOL_BF16, (e, ew, eS)


def test_decode_workload_1000_steps():
    w = gen.workload("decode")
    N, H, d = w.B, w.H, w.dk
    steps = 1000
    S = gen.decode_state(N, H, d, d, device="cuda")
    idx = np.random.default_rng(5).choice(N * H, size=64, replace=False)
    n_i, h_i = torch.as_tensor(idx // H), torch.as_tensor(idx % H)
    S_host = S[n_i, h_i].cpu().double().numpy()[:, None]  # [64, 1, d, d]
    worst = 0.0
    for step in range(steps):
        xs = gen.decode_step_inputs(N, H, d, d, step, device="cuda")
        o = kda.kda_decode_step(xs["q"], xs["k"], xs["v"], xs["log_alpha"], xs["beta"], S)
        sub = {k: v[n_i, h_i][:, None].cpu() for k, v in xs.items()}
        o_ref, S_host = oracle.decode(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"], S_host)
        e = max_rel_l2_per_slice(o[n_i, h_i].float().cpu().numpy(), o_ref[:, 0], slice_axes=(0,))
        worst = max(worst, e)
        assert e <= TOL_BF16, (step, e)
    assert kda.kda_check_device_error() == 0
    eS = max_rel_l2_per_slice(S[n_i, h_i].cpu().numpy(), S_host[:, 0], slice_axes=(0,))
    assert eS <= TOL_BF16, (eS, worst)
