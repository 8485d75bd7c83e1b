"""GPU parity of the serving-state variants (kda_chunk_fwd_slots,
kda_decode_step_slots) against the fp64 oracle.

The slot semantics are plain indexing, written out here on the host: the
initial state of sequence n is pool[slot[n]] (zeros when its slot is
negative or has_initial_state[n] is 0), the oracle runs the recurrence, and
the expected pool is the old pool with row slot[n] replaced by the final
state of sequence n for every non-negative slot.  Rows no sequence names
must come back bit-identical.  Tolerances are those of the dense calls.
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
KDA_ERR_ARGUMENT = -10


def _pool(num_slots, H, d, seed):
    return gen.decode_state(num_slots, H, d, d, seed=seed)


def _expected_prefill(x, pool, slots, has_init):
    """Oracle (o, pool) for a slot-indexed prefill."""
    N = len(slots)
    H, dk, dv = pool.shape[1], pool.shape[2], pool.shape[3]
    S0 = np.zeros((N, H, dk, dv))
    P = pool.double().numpy()
    for n, s in enumerate(slots):
        if s >= 0 and (has_init is None or has_init[n]):
            S0[n] = P[s]
    cu = None if x["cu_seqlens"] is None else x["cu_seqlens"].cpu().numpy()
    o_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S0, cu_seqlens=cu)
    P_ref = P.copy()
    for n, s in enumerate(slots):
        if s >= 0:
            P_ref[s] = S_ref[n]
    return o_ref, P_ref


def _run_prefill_slots(x, pool, slots, has_init, **kw):
    xd = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    pool_d = pool.cuda()
    slots_d = torch.tensor(slots, dtype=torch.int32, device="cuda")
    hi = None if has_init is None else torch.tensor(has_init, dtype=torch.uint8, device="cuda")
    o = kda.kda_chunk_fwd_slots(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], pool_d, slots_d, hi,
                                xd["cu_seqlens"], **kw)
    return o, pool_d


def _check_prefill(x, pool, slots, has_init, o, pool_d):
    o_ref, P_ref = _expected_prefill(x, pool, slots, has_init)
    o = o.float().cpu().numpy()
    P = pool_d.cpu().numpy()
    c = x["cu_seqlens"].cpu().numpy()
    err_o = err_w = 0.0
    for n in range(len(c) - 1):
        a, e = int(c[n]), int(c[n + 1])
        if e > a:
            err_o = max(err_o, max_rel_l2_per_slice(o[0, a:e], o_ref[0, a:e], slice_axes=(1,)))
            err_w = max(err_w, max_rel_l2_per_window(o[0, a:e], o_ref[0, a:e]))
    named = sorted({s for s in slots if s >= 0})
    untouched = [r for r in range(pool.shape[0]) if r not in named]
    assert np.array_equal(P[untouched], pool.numpy()[untouched]), "a row no sequence names was written"
    err_S = max_rel_l2_per_slice(P[named], P_ref[named], slice_axes=(0, 1))
    assert err_o <= TOL_BF16 and err_w <= TOL_BF16 and err_S <= TOL_BF16, (err_o, err_w, err_S)


# Packed batch: ragged tails, an empty sequence, a prompt crossing many
# chunks (900 tokens = 14 chunks + a 4-token tail), single tokens.
LENS = [130, 0, 900, 1, 64, 257, 70]
SLOTS = [7, 2, 0, -1, 9, 4, 5]          # a permutation of live slots, one padding row
HAS_INIT = [1, 1, 0, 1, 1, 0, 1]        # two new requests start from zeros


@pytest.mark.parametrize("recurrent", [False, True])
def test_prefill_slots_matches_oracle(recurrent):
    x = gen.make_inputs(1, sum(LENS), 3, 128, 128, seqlens=LENS, s0="none", seed=41)
    pool = _pool(11, 3, 128, seed=42)
    o, pool_d = _run_prefill_slots(x, pool, SLOTS, HAS_INIT, recurrent=recurrent)
    assert kda.kda_check_device_error() == 0
    _check_prefill(x, pool, SLOTS, HAS_INIT, o, pool_d)


def test_prefill_slots_resume_by_default():
    """has_initial_state omitted: every sequence resumes from its slot."""
    lens = [65, 200, 3]
    x = gen.make_inputs(1, sum(lens), 2, 128, 128, seqlens=lens, s0="none", seed=43)
    pool = _pool(4, 2, 128, seed=44)
    slots = [3, 0, 1]
    o, pool_d = _run_prefill_slots(x, pool, slots, None)
    assert kda.kda_check_device_error() == 0
    _check_prefill(x, pool, slots, None, o, pool_d)


def test_prefill_slots_bit_identical_to_dense_call():
    """Slot indexing moves states, never changes arithmetic: the slot call and
    kda_chunk_fwd with the gathered states give the same bits."""
    lens = [300, 64, 129]
    x = gen.make_inputs(1, sum(lens), 2, 128, 128, seqlens=lens, s0="none", seed=45)
    xd = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    pool = _pool(6, 2, 128, seed=46).cuda()
    slots = [4, 1, 5]
    S0 = pool[slots].contiguous()
    o_ref, S_ref = kda.kda_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], S0, xd["cu_seqlens"])
    o = kda.kda_chunk_fwd_slots(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], pool,
                                torch.tensor(slots, dtype=torch.int32, device="cuda"), None, xd["cu_seqlens"])
    assert torch.equal(o, o_ref) and torch.equal(pool[slots], S_ref)


def test_prefill_slots_chunked_prefill_resumes_cached_state():
    """A prompt prefilled in two calls through its slot (a cached prefix, then
    the rest with has_initial_state = 1) equals one call over the whole
    prompt; the split sits on a chunk boundary, so the bits match."""
    T, T1, H = 448, 192, 2
    x = gen.make_inputs(1, T, H, 128, 128, seqlens=[T], s0="none", seed=47)
    xd = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    one = torch.tensor([2], dtype=torch.int32, device="cuda")
    pool_a = torch.zeros(3, H, 128, 128, device="cuda")
    o_full = kda.kda_chunk_fwd_slots(xd["q"], xd["k"], xd["v"], xd["log_alpha"], xd["beta"], pool_a, one,
                                     torch.zeros(1, dtype=torch.uint8, device="cuda"),
                                     torch.tensor([0, T], dtype=torch.int32, device="cuda"))
    pool_b = torch.full((3, H, 128, 128), float("nan"), device="cuda")  # stale contents of a reused slot
    parts = []
    for a, b, init in ((0, T1, 0), (T1, T, 1)):
        sl = {k: xd[k][:, a:b].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")}
        parts.append(kda.kda_chunk_fwd_slots(sl["q"], sl["k"], sl["v"], sl["log_alpha"], sl["beta"], pool_b, one,
                                             torch.tensor([init], dtype=torch.uint8, device="cuda"),
                                             torch.tensor([0, b - a], dtype=torch.int32, device="cuda")))
    assert kda.kda_check_device_error() == 0
    assert torch.equal(torch.cat(parts, 1), o_full)
    assert torch.equal(pool_b[2], pool_a[2])


def test_prefill_slot_out_of_range_is_refused_on_device():
    lens = [70, 10]
    x = gen.make_inputs(1, sum(lens), 2, 128, 128, seqlens=lens, s0="none", seed=48)
    pool = _pool(3, 2, 128, seed=49)
    o, pool_d = _run_prefill_slots(x, pool, [1, 3], None)
    assert kda.kda_check_device_error() == KDA_ERR_ARGUMENT
    assert kda.kda_check_device_error() == 0
    # sequence 1 ran as padding (zero start, state dropped); sequence 0 as usual
    _check_prefill(x, pool, [1, -1], None, o, pool_d)


@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.float32)])
def test_decode_slots_matches_oracle(d, dtype):
    N, H, num_slots = 12, 3, 20
    rng = np.random.default_rng(50)
    pool = _pool(num_slots, H, d, seed=51)
    slots = rng.permutation(num_slots)[:N].astype(np.int32)
    slots[[3, 8]] = -1
    pool_d = pool.cuda()
    slots_d = torch.from_numpy(slots).cuda()
    P_ref = pool.double().numpy()
    tol = 1e-4 if dtype == torch.float32 else TOL_BF16
    for step in range(3):
        x = {k: v.cuda() for k, v in gen.decode_step_inputs(N, H, d, d, step, dtype=dtype, seed=52).items()}
        o = kda.kda_decode_step_slots(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool_d, slots_d)
        S_in = np.stack([P_ref[s] if s >= 0 else np.zeros((H, d, d)) for s in slots])
        o_ref, S_new = oracle.decode(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S_in)
        for n, s in enumerate(slots):
            if s >= 0:
                P_ref[s] = S_new[n]
        eo = max_rel_l2_per_slice(o.float().cpu().numpy(), o_ref, slice_axes=(0, 1))
        eS = max_rel_l2_per_slice(pool_d.cpu().numpy(), P_ref, slice_axes=(0, 1))
        assert eo <= tol and eS <= tol, (step, eo, eS)
    assert kda.kda_check_device_error() == 0
    untouched = sorted(set(range(num_slots)) - set(int(s) for s in slots))
    assert torch.equal(pool_d.cpu()[untouched], pool[untouched])


def test_decode_slots_bit_identical_to_dense_step():
    N, H, d = 16, 2, 128
    pool = _pool(N + 5, H, d, seed=53).cuda()
    slots = torch.randperm(N + 5, generator=torch.Generator().manual_seed(54))[:N].to(torch.int32).cuda()
    S = pool[slots.long()].clone()
    x = {k: v.cuda() for k, v in gen.decode_step_inputs(N, H, d, d, 0, seed=55).items()}
    o_ref = kda.kda_decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S)
    o = kda.kda_decode_step_slots(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, slots)
    assert torch.equal(o, o_ref) and torch.equal(pool[slots.long()], S)


def test_decode_slot_out_of_range_is_refused_on_device():
    N, H, d = 4, 2, 128
    pool = _pool(4, H, d, seed=56).cuda()
    before = pool.clone()
    slots = torch.tensor([0, 4, 1000, 2], dtype=torch.int32, device="cuda")
    x = {k: v.cuda() for k, v in gen.decode_step_inputs(N, H, d, d, 0, seed=57).items()}
    kda.kda_decode_step_slots(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, slots)
    assert kda.kda_check_device_error() == KDA_ERR_ARGUMENT
    assert torch.equal(pool[[1, 3]], before[[1, 3]])
