"""The C ABI boundary, checked on the host (no GPU needed).

The library must load, export every entry point include/kda.h declares, and
reject bad arguments with the documented status *before* launching anything.
Only argument errors that are detected ahead of any CUDA call are exercised
here, so no test ever hands a kernel a bogus pointer.
"""
import ctypes
import re
from pathlib import Path

import pytest

import gated_delta_rule_110_b200 as kda

ROOT = Path(__file__).resolve().parents[1]


def declared_functions():
    text = (ROOT / "include" / "kda.h").read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z_]+)\s*\(", text)))


def test_header_declares_the_expected_entry_points():
    assert declared_functions() == sorted(kda.EXPORTED_SYMBOLS)


def test_library_loads_and_exports_every_declared_symbol():
    lib = kda.load_library()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert kda.kda_abi_version() == 7


def test_status_strings():
    for code in range(0, -11, -1):
        s = kda.kda_status_string(code)
        assert isinstance(s, str) and s and s != "unknown status"
    assert kda.kda_status_string(-99) == "unknown status"


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails validation first


def call_fwd(shape, ptrs=None, ws=None, ws_bytes=0):
    lib = kda.load_library()
    p = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, S0=None, cu=None, o=FAKE, ST=None)
    p.update(ptrs or {})
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.kda_chunk_fwd(ctypes.byref(shape), vp(p["q"]), vp(p["k"]), vp(p["v"]), vp(p["la"]),
                             vp(p["beta"]), vp(p["S0"]), vp(p["cu"]), vp(p["o"]), vp(p["ST"]), vp(ws), ws_bytes,
                             None)


def tc_shape(**kw):
    base = dict(B=1, T=128, H=2, dk=128, dv=128, chunk=64, n_seqs=0, io_dtype=1, gate_dtype=1, flags=0)
    base.update(kw)
    return kda.make_shape(**base)


def test_null_shape():
    lib = kda.load_library()
    assert lib.kda_chunk_fwd(None, *([None] * 9), None, 0, None) == -1
    assert lib.kda_decode_step(None, *([None] * 7), None) == -1
    assert lib.kda_chunk_fwd_workspace_size(None) == 0


@pytest.mark.parametrize("field,value,status", [
    ("io_dtype", 7, -3), ("gate_dtype", -1, -3), ("B", 0, -2), ("H", 0, -2), ("T", -1, -2),
    ("dk", 96, -5), ("dv", 32, -5), ("chunk", 48, -5), ("chunk", 32, -5), ("chunk", 16, -5),
    ("flags", 0x80, -10), ("flags", 0x2, -10),
])
def test_bad_shape_fields(field, value, status):
    assert call_fwd(tc_shape(**{field: value})) == status


def test_null_inputs_and_misalignment():
    assert call_fwd(tc_shape(), {"q": None}) == -1
    assert call_fwd(tc_shape(), {"o": None}) == -1
    assert call_fwd(tc_shape(), {"k": FAKE + 2}) == -4
    assert call_fwd(tc_shape(), {"beta": FAKE + 1}) == -4
    assert call_fwd(tc_shape(), {"S0": FAKE + 8}) == -4


def test_workspace_required_on_tensor_core_path():
    # without a workspace the call is refused (KDA_ERR_WORKSPACE), or, on a
    # machine without a GPU, fails while sizing the launch (KDA_ERR_CUDA)
    assert call_fwd(tc_shape(B=2, T=200)) in (-6, -7)


def test_cuda_core_paths_need_no_workspace():
    assert kda.kda_chunk_fwd_workspace_size(tc_shape(io_dtype=0)) == 0
    assert kda.kda_chunk_fwd_workspace_size(tc_shape(dk=64, dv=64)) == 0
    assert kda.kda_chunk_fwd_workspace_size(tc_shape(flags=kda.KDA_FLAG_PATH_RECURRENT)) == 0


def test_tuning_flags_are_accepted_and_encoded():
    assert kda.tuning_flags(3, 10) == (3 << 8) | (10 << 16)
    with pytest.raises(ValueError):
        kda.tuning_flags(256, 0)
    # the flag bits pass validation (the call then fails on the missing workspace,
    # or on the absent device, never on the flags)
    assert call_fwd(tc_shape(flags=kda.tuning_flags(2, 8))) in (-6, -7)


@pytest.mark.gpu
def test_pipelined_path_workspace_is_bounded_by_the_sm_count():
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    small = kda.kda_chunk_fwd_workspace_size(tc_shape())
    big = kda.kda_chunk_fwd_workspace_size(tc_shape(B=1, T=1 << 20, H=64))
    assert 0 < small <= big <= sms * 16 * 66560 + 65536
    capped = kda.kda_chunk_fwd_workspace_size(tc_shape(H=64, flags=kda.tuning_flags(3, 0)))
    assert capped < 4 * 16 * 66560 + 65536


def test_packed_requires_single_batch_row():
    assert call_fwd(tc_shape(B=2, n_seqs=3), {"cu": FAKE}) == -2


def test_decode_rejects_multi_token():
    lib = kda.load_library()
    s = kda.make_shape(4, 2, 2, 128, 128)
    args = [ctypes.c_void_p(FAKE)] * 7
    assert lib.kda_decode_step(ctypes.byref(s), *args, None) == -2


def call_fwd_slots(shape, pool=FAKE, num_slots=4, slots=FAKE, has_init=None, cu=None):
    lib = kda.load_library()
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    f = vp(FAKE)
    return lib.kda_chunk_fwd_slots(ctypes.byref(shape), f, f, f, f, f, vp(pool), num_slots, vp(slots),
                                   vp(has_init), vp(cu), f, None, 0, None)


def test_slot_prefill_host_validation():
    assert call_fwd_slots(tc_shape(), pool=None) == -1
    assert call_fwd_slots(tc_shape(), slots=None) == -1
    assert call_fwd_slots(tc_shape(), num_slots=0) == -2
    assert call_fwd_slots(tc_shape(), slots=FAKE + 2) == -4
    assert call_fwd_slots(tc_shape(), pool=FAKE + 8) == -4
    assert call_fwd_slots(tc_shape(chunk=32)) == -5
    # the CUDA-core path needs no workspace: it gets as far as the launch
    # (which fails on a machine without a GPU)
    assert call_fwd_slots(tc_shape(B=2, T=200)) in (-6, -7)


def test_slot_decode_host_validation():
    lib = kda.load_library()
    f = ctypes.c_void_p(FAKE)
    call = lambda shape, pool, n, slots: lib.kda_decode_step_slots(ctypes.byref(shape), f, f, f, f, f, pool, n,
                                                                   slots, f, None)
    s1 = kda.make_shape(4, 1, 2, 128, 128)
    assert call(s1, f, 4, None) == -1
    assert call(s1, None, 4, f) == -1
    assert call(s1, f, 0, f) == -2
    assert call(kda.make_shape(4, 2, 2, 128, 128), f, 4, f) == -2
    assert call(s1, f, 4, ctypes.c_void_p(FAKE + 2)) == -4


def call_fwd_gated(shape, gate=FAKE, weight=FAKE, eps=1e-5):
    lib = kda.load_library()
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    f = vp(FAKE)
    return lib.kda_chunk_fwd_gated(ctypes.byref(shape), f, f, f, f, f, None, None, vp(gate), vp(weight),
                                   ctypes.c_float(eps), f, None, None, 0, None)


def test_gated_prefill_host_validation():
    assert call_fwd_gated(tc_shape(), gate=None) == -1
    assert call_fwd_gated(tc_shape(), weight=None) == -1
    assert call_fwd_gated(tc_shape(), eps=-1.0) == -10
    assert call_fwd_gated(tc_shape(), eps=float("nan")) == -10
    assert call_fwd_gated(tc_shape(), eps=float("inf")) == -10
    assert call_fwd_gated(tc_shape(), gate=FAKE + 2) == -4
    assert call_fwd_gated(tc_shape(), weight=FAKE + 4) == -4
    assert call_fwd_gated(tc_shape(flags=kda.KDA_FLAG_GATE_FUSED | kda.KDA_FLAG_GATE_SEPARATE)) == -10
    # every path takes the epilogue: these get as far as the launch (which
    # fails on a machine without a GPU)
    for shape in (tc_shape(io_dtype=0), tc_shape(dk=64, dv=64), tc_shape(flags=kda.KDA_FLAG_PATH_RECURRENT),
                  tc_shape(B=2, T=200), tc_shape(flags=kda.KDA_FLAG_GATE_SEPARATE)):
        assert call_fwd_gated(shape) in (-6, -7)


def call_fwd_layer(shape, A=FAKE, bias=FAKE, gate=None, weight=None, eps=1e-5):
    lib = kda.load_library()
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    f = vp(FAKE)
    return lib.kda_chunk_fwd_layer(ctypes.byref(shape), f, f, f, f, vp(A), vp(bias), f, None, None, vp(gate),
                                   vp(weight), ctypes.c_float(eps), f, None, None, 0, None)


def test_layer_prefill_host_validation():
    assert call_fwd_layer(tc_shape(), A=None) == -1
    assert call_fwd_layer(tc_shape(), bias=None) == -1
    assert call_fwd_layer(tc_shape(), A=FAKE + 2) == -4
    assert call_fwd_layer(tc_shape(), bias=FAKE + 4) == -4
    assert call_fwd_layer(tc_shape(), gate=FAKE) == -1
    assert call_fwd_layer(tc_shape(), weight=FAKE) == -1
    assert call_fwd_layer(tc_shape(), gate=FAKE, weight=FAKE, eps=-1.0) == -10
    assert call_fwd_layer(tc_shape(), gate=FAKE + 2, weight=FAKE) == -4
    # the tensor-core kernel takes a bf16 gate projection only; the CUDA-core
    # paths take any (they get as far as the launch)
    assert call_fwd_layer(tc_shape(gate_dtype=0)) == -5
    for shape in (tc_shape(io_dtype=0), tc_shape(dk=64, dv=64), tc_shape(flags=kda.KDA_FLAG_PATH_RECURRENT)):
        assert call_fwd_layer(shape) in (-6, -7)
    assert call_fwd_layer(tc_shape(B=2, T=200)) in (-6, -7)
    assert call_fwd_layer(tc_shape(B=2, T=200), gate=FAKE, weight=FAKE) in (-6, -7)


def test_python_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 1, 64)
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd(x, x, x, x, torch.zeros(1, 4, 1))


def test_layer_decode_host_validation():
    lib = kda.load_library()
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    f = vp(FAKE)
    s1 = kda.make_shape(4, 1, 2, 128, 128)
    call = lambda shape, A=FAKE, bias=FAKE, slots=None, n=0, gate=None, w=None, eps=1e-5: lib.kda_decode_step_layer(
        ctypes.byref(shape), f, f, f, f, vp(A), vp(bias), f, f, vp(slots), n, vp(gate), vp(w), ctypes.c_float(eps),
        f, None)
    assert call(s1, A=None) == -1
    assert call(s1, bias=None) == -1
    assert call(s1, A=FAKE + 2) == -4
    assert call(s1, slots=FAKE, n=0) == -2
    assert call(s1, gate=FAKE) == -1
    assert call(s1, gate=FAKE, w=FAKE, eps=-1.0) == -10
    assert call(kda.make_shape(4, 2, 2, 128, 128)) == -2


def test_prefill_plan_on_a_148_sm_device():
    """The host's plan for the benchmark workloads on a 148-SM B200: state /
    transform split, where the output epilogue goes, ring depth and
    workspace (host-only: no device is touched with num_sms given)."""
    from gated_delta_rule_110_b200 import inputs as gen
    def plan(name, flags=0):
        w = gen.workload(name)
        n = 0 if w.seqlens is None else len(w.seqlens)
        return kda.kda_prefill_plan(kda.make_shape(w.B, w.T, w.H, w.dk, w.dv, 64, n, 1, 1, flags), 148)
    pre, var, lng = plan("prefill"), plan("varlen"), plan("long")
    # 64 chains: one per state CTA, the other 84 CTAs transform (state side 1 chain, transform 128 / 84)
    assert (pre["state_ctas"], pre["grid_ctas"]) == (64, 148)
    # 256 chains: R balances ceil(256 / R) against 512 / (148 - R)
    assert var["state_ctas"] == 52
    assert lng["state_ctas"] == 32
    # the epilogue is fused where the transform side bounds the call
    assert pre["fuse_output_gate"] == 1 and var["fuse_output_gate"] == 1 and lng["fuse_output_gate"] == 0
    assert plan("long", kda.KDA_FLAG_GATE_FUSED)["fuse_output_gate"] == 1
    assert plan("prefill", kda.KDA_FLAG_GATE_SEPARATE)["fuse_output_gate"] == 0
    for p in (pre, var, lng):
        slot_bytes = p["state_ctas"] * 66560
        assert 4 <= p["ring_depth"] <= 16
        assert p["workspace_bytes"] >= p["ring_depth"] * slot_bytes
        assert p["min_workspace_bytes"] < p["workspace_bytes"]
        assert p["ring_depth"] == 4 or p["ring_depth"] * slot_bytes <= 48 << 20
    # overrides through the flags
    assert plan("prefill", kda.tuning_flags(16, 0))["state_ctas"] == 16
    assert plan("prefill", kda.tuning_flags(0, 100))["grid_ctas"] == 100


def test_prefill_plan_refuses_other_paths():
    lib = kda.load_library()
    info = kda.PrefillPlanInfo()
    assert lib.kda_prefill_plan(ctypes.byref(tc_shape(io_dtype=0)), 148, ctypes.byref(info)) == -5
    assert lib.kda_prefill_plan(ctypes.byref(tc_shape()), 148, None) == -1
    assert lib.kda_prefill_plan(None, 148, ctypes.byref(info)) == -1


def test_python_binding_checks_shapes_before_the_device():
    """Argument errors of the gated, layer and decode-layer calls are reported
    as such (before the no-CPU-path check), so they surface on any machine."""
    import torch
    q = torch.zeros(1, 8, 2, 128)
    beta = torch.zeros(1, 8, 2)
    A, bias = torch.zeros(2), torch.zeros(2, 128)
    with pytest.raises(ValueError, match="out_gate"):
        kda.kda_chunk_fwd_gated(q, q, q, q, beta, torch.zeros(1, 8, 2, 64), torch.zeros(128))
    with pytest.raises(ValueError, match="norm_weight"):
        kda.kda_chunk_fwd_gated(q, q, q, q, beta, q, torch.zeros(64))
    with pytest.raises(ValueError, match="gate_mode"):
        kda.kda_chunk_fwd_gated(q, q, q, q, beta, q, torch.zeros(128), gate_mode="sometimes")
    with pytest.raises(ValueError, match="gate_f"):
        kda.kda_chunk_fwd_layer(q, q, q, torch.zeros(1, 8, 2, 64), A, bias, beta)
    with pytest.raises(ValueError, match="A_log"):
        kda.kda_chunk_fwd_layer(q, q, q, q, torch.zeros(3), bias, beta)
    with pytest.raises(ValueError, match="go together"):
        kda.kda_chunk_fwd_layer(q, q, q, q, A, bias, beta, out_gate=q)
    with pytest.raises(ValueError, match="A_log"):
        kda.kda_decode_step_layer(q[:, 0], q[:, 0], q[:, 0], q[:, 0], torch.zeros(5), bias, beta[:, 0],
                                  torch.zeros(1, 2, 128, 128))
    with pytest.raises(ValueError, match="CUDA"):
        kda.kda_chunk_fwd_layer(q, q, q, q, A, bias, beta)
