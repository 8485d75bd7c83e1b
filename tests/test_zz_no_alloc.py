"""kda_chunk_fwd_noalloc: the prefill for callers that cannot allocate.

Some users of this library run the prefill where they have no way to get
device memory: a plugin inside a framework whose memory pool already owns the
GPU and exposes no allocator across the C boundary, or a serving loop that
bans cudaMalloc because it synchronises the whole device.  For them the
library offers kda_chunk_fwd_noalloc, which runs the same tensor-core path as
kda_chunk_fwd with that path's workspace (its operand ring and counters) in a
fixed 64 MiB array inside the library instead of a caller-supplied buffer.

These tests call it through the C ABI and check it against kda_chunk_fwd and
against the fp64 oracle, within the bf16 tolerance the other parity tests use,
on two calls in a row with different inputs: the second call also shows that
what the first left in the shared array does not leak into its result.  A
separate test runs kda_chunk_fwd with a workspace filled with NaN bytes: a
finite, correct result shows the kernels never read a workspace byte they did
not write in the same call, which is what makes sharing one array safe.  The
file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import gated_delta_rule_110_b200 as kda
import oracle
from gated_delta_rule_110_b200 import inputs as gen

TOL_BF16 = 2e-2


def _rel_slices(x, ref, axes):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    other = tuple(a for a in range(x.ndim) if a not in axes)
    num = np.sqrt(((x - ref) ** 2).sum(axis=other))
    den = np.maximum(np.sqrt((ref ** 2).sum(axis=other)), 1e-30)
    return float((num / den).max())


def _call_noalloc_c_abi(x, o, S_T):
    lib = kda.load_library()
    B, T, H, dk = x["q"].shape
    n_seqs = 0 if x["cu_seqlens"] is None else x["cu_seqlens"].numel() - 1
    shape = kda.make_shape(B, T, H, dk, x["v"].shape[-1], 64, n_seqs, kda.KDA_BF16, kda.KDA_BF16)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.kda_chunk_fwd_noalloc(ctypes.byref(shape), p(x["q"]), p(x["k"]), p(x["v"]), p(x["log_alpha"]),
                                     p(x["beta"]), p(x["S0"]), p(x["cu_seqlens"]), p(o), p(S_T), stream)


def _cases():
    return [
        gen.make_inputs(2, 200, 3, 128, 128, seed=301),                        # batched, ragged tail
        gen.make_inputs(1, 330, 2, 128, 128, seqlens=[130, 1, 199], seed=302),  # packed sequences
    ]


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_and_oracle_on_two_calls():
    for x in _cases():
        xd = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
        o_ref, S_ref = kda.kda_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["S0"],
                                         xd["cu_seqlens"])
        o = torch.full_like(xd["v"], float("nan"))
        S_T = torch.full_like(S_ref, float("nan"))
        rc = _call_noalloc_c_abi(xd, o, S_T)
        assert rc == 0, kda.kda_status_string(rc)
        assert kda.kda_check_device_error() == 0
        assert _rel_slices(o.float().cpu(), o_ref.float().cpu(), (0, 2)) <= TOL_BF16
        assert _rel_slices(S_T.cpu(), S_ref.cpu(), (0, 1)) <= TOL_BF16
        cu = None if x["cu_seqlens"] is None else x["cu_seqlens"].numpy()
        o_or, S_or = oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], cu_seqlens=cu)
        o_h = o.float().cpu().numpy()
        if cu is None:
            assert _rel_slices(o_h, o_or, (0, 2)) <= TOL_BF16
        else:
            for n in range(len(cu) - 1):
                a, b = int(cu[n]), int(cu[n + 1])
                assert _rel_slices(o_h[:, a:b], o_or[:, a:b], (0, 2)) <= TOL_BF16
        assert _rel_slices(S_T.cpu().numpy(), S_or, (0, 1)) <= TOL_BF16


@pytest.mark.gpu
def test_workspace_bytes_are_written_before_they_are_read():
    x = _cases()[1]
    xd = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    shape = kda.make_shape(1, xd["q"].shape[1], 2, 128, 128, 64, 3, kda.KDA_BF16, kda.KDA_BF16)
    ws = torch.full((kda.kda_chunk_fwd_workspace_size(shape),), 0xFF, dtype=torch.uint8, device="cuda")
    o, S = kda.kda_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["S0"], xd["cu_seqlens"],
                             workspace=ws)
    assert kda.kda_check_device_error() == 0
    assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
    o_or, S_or = oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"],
                                cu_seqlens=x["cu_seqlens"].numpy())
    assert _rel_slices(S.cpu().numpy(), S_or, (0, 1)) <= TOL_BF16


@pytest.mark.gpu
def test_noalloc_runs_the_deepest_ring_its_array_holds():
    """147 state CTAs: the 64 MiB array holds a 6-slot ring (a 16-slot ring
    would need ~156 MB), which the call uses; the result matches the workspace
    entry point given its preferred workspace (a different ring depth: the
    ring depth changes no arithmetic)."""
    x = gen.make_inputs(1, 64, 148, 128, 128, seed=303)
    xd = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    flags = kda.tuning_flags(147, 0)
    shape = kda.make_shape(1, 64, 148, 128, 128, 64, 0, kda.KDA_BF16, kda.KDA_BF16, flags)
    slot_bytes = 66560
    assert 16 * 147 * slot_bytes > kda_noalloc_bytes() > 2 * 147 * slot_bytes
    o_ref, S_ref = kda.kda_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], xd["S0"],
                                     state_ctas=147)
    o, S_T = torch.empty_like(o_ref), torch.empty_like(S_ref)
    lib = kda.load_library()
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = lib.kda_chunk_fwd_noalloc(ctypes.byref(shape), p(xd["q"]), p(xd["k"]), p(xd["v"]), p(xd["log_alpha"]),
                                   p(xd["beta"]), p(xd["S0"]), None, p(o), p(S_T),
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, kda.kda_status_string(rc)
    assert kda.kda_check_device_error() == 0
    assert torch.equal(o, o_ref) and torch.equal(S_T, S_ref)


def kda_noalloc_bytes():
    return 64 * 1024 * 1024


def test_noalloc_validates_before_touching_the_device():
    """Invalid shapes are refused on the host with the documented status,
    without a GPU."""
    lib = kda.load_library()
    fake = ctypes.c_void_p(0x10000)
    assert lib.kda_chunk_fwd_noalloc(None, fake, fake, fake, fake, fake, None, None, fake, None, None) == -1
    bad = kda.make_shape(1, 128, 2, 128, 128, 32, 0, kda.KDA_BF16, kda.KDA_BF16)
    assert lib.kda_chunk_fwd_noalloc(ctypes.byref(bad), fake, fake, fake, fake, fake, None, None, fake, None,
                                     None) == -5
