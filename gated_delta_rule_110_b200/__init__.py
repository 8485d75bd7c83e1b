"""B200-native Kimi Delta Attention (KDA) operator.

Python binding of ``libkda.so`` (the C ABI in ``include/kda.h``): argument
marshalling only.  PyTorch supplies device memory and the current CUDA
stream; every step of the operator runs in the library's sm_100a kernels.
There is no CPU or PyTorch fallback: if the library cannot be loaded, or a
tensor is not on a CUDA device, the call raises.

Entry points (same names as the C ABI):

* ``kda_chunk_fwd(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None)``
  chunkwise-parallel prefill -> ``(o, S_T)``
* ``kda_decode_step(q, k, v, log_alpha, beta, S)`` one recurrent token per
  (sequence, head), ``S`` updated in place -> ``o``
* ``kda_chunk_fwd_layer(q, k, v, gate_f, A_log, dt_bias, beta, ...)`` raw q, k and
  the decay gate's projection in (L2 norm and gate computed in the kernel) -> ``(o, S_T)``
* ``kda_decode_step_layer(q, k, v, gate_f, A_log, dt_bias, beta, state, ...)`` one
  decode step with the layer's producer steps (and optional output epilogue)
* ``kda_chunk_fwd_gated(q, k, v, log_alpha, beta, out_gate, norm_weight, ...)``
  prefill followed by the per-head RMSNorm and sigmoid output gate -> ``(o', S_T)``
* ``kda_chunk_fwd_slots(q, k, v, log_alpha, beta, state_pool, state_slots,
  has_initial_state=None, cu_seqlens=None)`` prefill reading and writing the
  states in place in a slot-indexed pool -> ``o``
* ``kda_decode_step_slots(q, k, v, log_alpha, beta, state_pool, state_slots)``
  decode step on a slot-indexed pool -> ``o``
* ``kda_chunk_fwd_noalloc(...)`` kda_chunk_fwd on the library's own scratch array
* ``kda_chunk_fwd_workspace_size(...)``, ``kda_prefill_plan(shape, num_sms)``,
  ``kda_check_device_error()``, ``kda_status_string(code)``, ``kda_abi_version()``

Sharded variants (one batch across the ranks of a process group) are in
``gated_delta_rule_110_b200.shard``.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libkda.so"

KDA_OK = 0
KDA_F32, KDA_BF16 = 0, 1
KDA_FLAG_VALIDATE_CU_SEQLENS = 0x1
KDA_FLAG_PATH_RECURRENT = 0x4
KDA_FLAG_GATE_FUSED = 0x8
KDA_FLAG_GATE_SEPARATE = 0x10
_GATE_MODES = {"auto": 0, "fused": KDA_FLAG_GATE_FUSED, "separate": KDA_FLAG_GATE_SEPARATE}

_STATUS_NAMES = {
    0: "KDA_OK", -1: "KDA_ERR_NULL", -2: "KDA_ERR_SHAPE", -3: "KDA_ERR_DTYPE", -4: "KDA_ERR_ALIGN",
    -5: "KDA_ERR_UNSUPPORTED", -6: "KDA_ERR_WORKSPACE", -7: "KDA_ERR_CUDA", -8: "KDA_ERR_TIMEOUT",
    -9: "KDA_ERR_INTERNAL", -10: "KDA_ERR_ARGUMENT",
}

EXPORTED_SYMBOLS = (
    "kda_chunk_fwd_workspace_size", "kda_prefill_plan", "kda_chunk_fwd", "kda_chunk_fwd_gated",
    "kda_chunk_fwd_layer",
    "kda_chunk_fwd_noalloc",
    "kda_chunk_fwd_slots",
    "kda_decode_step", "kda_decode_step_slots", "kda_decode_step_layer", "kda_check_device_error", "kda_status_string",
    "kda_abi_version",
)


class KdaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_STATUS_NAMES.get(status, status)} ({kda_status_string(status)})")


class kda_shape(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("T", ctypes.c_int32), ("H", ctypes.c_int32),
        ("dk", ctypes.c_int32), ("dv", ctypes.c_int32), ("chunk", ctypes.c_int32),
        ("n_seqs", ctypes.c_int32), ("io_dtype", ctypes.c_int32), ("gate_dtype", ctypes.c_int32),
        ("flags", ctypes.c_uint32),
    ]


_lib = None


def load_library(build_if_missing: bool = True):
    """Load libkda.so (building it in-tree with nvcc if it is absent or stale)."""
    global _lib
    if _lib is not None:
        return _lib
    if build_if_missing:
        from . import build as _build
        try:
            _build.build()
        except Exception as exc:  # no nvcc: only an existing library can be used
            if not LIB_PATH.exists():
                raise RuntimeError(f"libkda.so is missing and could not be built: {exc}") from exc
    if not LIB_PATH.exists():
        raise RuntimeError(f"libkda.so not found at {LIB_PATH}")
    lib = ctypes.CDLL(str(LIB_PATH))
    vp, sp = ctypes.c_void_p, ctypes.POINTER(kda_shape)
    lib.kda_chunk_fwd_workspace_size.argtypes = [sp]
    lib.kda_chunk_fwd_workspace_size.restype = ctypes.c_size_t
    lib.kda_chunk_fwd.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.kda_chunk_fwd.restype = ctypes.c_int
    lib.kda_chunk_fwd_gated.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp,
                                        ctypes.c_size_t, vp]
    lib.kda_chunk_fwd_gated.restype = ctypes.c_int
    lib.kda_chunk_fwd_layer.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp,
                                        ctypes.c_size_t, vp]
    lib.kda_chunk_fwd_layer.restype = ctypes.c_int
    lib.kda_decode_step_layer.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int32, vp, vp,
                                          ctypes.c_float, vp, vp]
    lib.kda_decode_step_layer.restype = ctypes.c_int
    lib.kda_prefill_plan.argtypes = [sp, ctypes.c_int32, ctypes.POINTER(PrefillPlanInfo)]
    lib.kda_prefill_plan.restype = ctypes.c_int
    lib.kda_chunk_fwd_noalloc.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.kda_chunk_fwd_noalloc.restype = ctypes.c_int
    lib.kda_chunk_fwd_slots.argtypes = [sp, vp, vp, vp, vp, vp, vp, ctypes.c_int32, vp, vp, vp, vp, vp,
                                        ctypes.c_size_t, vp]
    lib.kda_chunk_fwd_slots.restype = ctypes.c_int
    lib.kda_decode_step.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.kda_decode_step.restype = ctypes.c_int
    lib.kda_decode_step_slots.argtypes = [sp, vp, vp, vp, vp, vp, vp, ctypes.c_int32, vp, vp, vp]
    lib.kda_decode_step_slots.restype = ctypes.c_int
    lib.kda_check_device_error.argtypes = [vp]
    lib.kda_check_device_error.restype = ctypes.c_int
    lib.kda_status_string.argtypes = [ctypes.c_int]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_abi_version.argtypes = []
    lib.kda_abi_version.restype = ctypes.c_int32
    _lib = lib
    return lib


def kda_status_string(status: int) -> str:
    return load_library().kda_status_string(int(status)).decode()


def kda_abi_version() -> int:
    return int(load_library().kda_abi_version())


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError(f"unsupported dtype {t.dtype}: use torch.bfloat16 or torch.float32")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors (the library has no CPU path)")
        if t is not None and not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")


def make_shape(B, T, H, dk, dv, chunk=64, n_seqs=0, io_dtype=KDA_BF16, gate_dtype=KDA_BF16, flags=0):
    return kda_shape(B, T, H, dk, dv, chunk, n_seqs, io_dtype, gate_dtype, flags)


def kda_chunk_fwd_workspace_size(shape: kda_shape) -> int:
    return int(load_library().kda_chunk_fwd_workspace_size(ctypes.byref(shape)))


def tuning_flags(state_ctas: int = 0, grid_ctas: int = 0) -> int:
    """Flag bits fixing the number of state CTAs / capping the grid of the
    pipelined tensor-core path (0 = automatic), as in include/kda.h."""
    if not (0 <= state_ctas <= 255 and 0 <= grid_ctas <= 255):
        raise ValueError("state_ctas and grid_ctas must be in [0, 255]")
    return (state_ctas << 8) | (grid_ctas << 16)


def _shape_of(q, v, log_alpha, cu_seqlens, chunk, validate, recurrent=False, state_ctas=0, grid_ctas=0):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    n_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    flags = (KDA_FLAG_VALIDATE_CU_SEQLENS if validate else 0) | (KDA_FLAG_PATH_RECURRENT if recurrent else 0)
    flags |= tuning_flags(state_ctas, grid_ctas)
    return make_shape(B, T, H, dk, dv, chunk, n_seqs, _dtype_code(q), _dtype_code(log_alpha), flags)


def kda_chunk_fwd(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, *, chunk: int = 64, o=None, S_T=None,
                  workspace=None, stream=None, validate: bool = False, output_final_state: bool = True,
                  recurrent: bool = False, state_ctas: int = 0, grid_ctas: int = 0):
    """Chunkwise KDA prefill.  Shapes as in include/kda.h; returns (o, S_T).

    The tensor-core path needs a workspace (allocated here from PyTorch's
    caching allocator if not given).  ``recurrent=True`` runs the fp32
    token-by-token CUDA-core recurrence instead (a reference path);
    ``state_ctas`` / ``grid_ctas`` override the tensor-core path's CTA split
    (0 = automatic)."""
    import torch
    _need_cuda(q, k, v, log_alpha, beta, S0, cu_seqlens, o, S_T, workspace)
    shape = _shape_of(q, v, log_alpha, cu_seqlens, chunk, validate, recurrent, state_ctas, grid_ctas)
    N = shape.B if cu_seqlens is None else shape.n_seqs
    if o is None:
        o = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    if S_T is None and output_final_state:
        S_T = torch.empty((N, shape.H, shape.dk, shape.dv), dtype=torch.float32, device=q.device)
    need = kda_chunk_fwd_workspace_size(shape)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load_library().kda_chunk_fwd(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
        _ptr(cu_seqlens), _ptr(o), _ptr(S_T), _ptr(workspace), ws_bytes, _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd")
    return o, S_T


def kda_chunk_fwd_gated(q, k, v, log_alpha, beta, out_gate, norm_weight, S0=None, cu_seqlens=None, *,
                        eps: float = 1e-5, chunk: int = 64, o=None, S_T=None, workspace=None, stream=None,
                        validate: bool = False, output_final_state: bool = True, recurrent: bool = False,
                        gate_mode: str = "auto", state_ctas: int = 0, grid_ctas: int = 0):
    """Prefill followed by the per-head RMSNorm and sigmoid output gate
    (include/kda.h, kda_chunk_fwd_gated): returns (o', S_T) with
    o' = o / rms(o) * norm_weight * sigmoid(out_gate).  ``gate_mode``:
    "auto" (the library decides), "fused" (in the tensor-core kernel's output
    warps) or "separate" (a pass over o after the prefill)."""
    import torch
    if out_gate.shape != v.shape or out_gate.dtype != v.dtype:
        raise ValueError("out_gate must have the shape and dtype of v")
    if norm_weight.dtype != torch.float32 or norm_weight.numel() != v.shape[-1]:
        raise ValueError("norm_weight must be a float32 tensor of dv values")
    if gate_mode not in _GATE_MODES:
        raise ValueError(f"gate_mode must be one of {sorted(_GATE_MODES)}")
    _need_cuda(q, k, v, log_alpha, beta, out_gate, norm_weight, S0, cu_seqlens, o, S_T, workspace)
    shape = _shape_of(q, v, log_alpha, cu_seqlens, chunk, validate, recurrent, state_ctas, grid_ctas)
    shape.flags |= _GATE_MODES[gate_mode]
    N = shape.B if cu_seqlens is None else shape.n_seqs
    if o is None:
        o = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    if S_T is None and output_final_state:
        S_T = torch.empty((N, shape.H, shape.dk, shape.dv), dtype=torch.float32, device=q.device)
    need = kda_chunk_fwd_workspace_size(shape)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load_library().kda_chunk_fwd_gated(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(cu_seqlens),
        _ptr(out_gate), _ptr(norm_weight), float(eps), _ptr(o), _ptr(S_T), _ptr(workspace), ws_bytes,
        _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd_gated")
    return o, S_T


def kda_chunk_fwd_layer(q, k, v, gate_f, A_log, dt_bias, beta, S0=None, cu_seqlens=None, *, out_gate=None,
                        norm_weight=None, eps: float = 1e-5, chunk: int = 64, o=None, S_T=None, workspace=None,
                        stream=None, validate: bool = False, output_final_state: bool = True,
                        recurrent: bool = False, gate_mode: str = "auto", state_ctas: int = 0, grid_ctas: int = 0):
    """The operator with the Kimi Linear layer's producer steps fused (raw q,
    k are L2-normalised, log alpha = -exp(A_log) * softplus(gate_f + dt_bias))
    and, with ``out_gate`` / ``norm_weight``, its output epilogue
    (include/kda.h, kda_chunk_fwd_layer).  Returns (o, S_T)."""
    import torch
    H, dk = q.shape[2], q.shape[3]
    if gate_f.shape != q.shape or gate_f.dtype != q.dtype:
        raise ValueError("gate_f must have the shape and dtype of q")
    if A_log.dtype != torch.float32 or A_log.numel() != H or dt_bias.dtype != torch.float32 or dt_bias.numel() != H * dk:
        raise ValueError("A_log must be float32 [H] and dt_bias float32 [H, dk]")
    if (out_gate is None) != (norm_weight is None):
        raise ValueError("out_gate and norm_weight go together")
    if out_gate is not None:
        if out_gate.shape != v.shape or out_gate.dtype != v.dtype:
            raise ValueError("out_gate must have the shape and dtype of v")
        if norm_weight.dtype != torch.float32 or norm_weight.numel() != v.shape[-1]:
            raise ValueError("norm_weight must be a float32 tensor of dv values")
    if gate_mode not in _GATE_MODES:
        raise ValueError(f"gate_mode must be one of {sorted(_GATE_MODES)}")
    _need_cuda(q, k, v, gate_f, A_log, dt_bias, beta, S0, cu_seqlens, out_gate, norm_weight, o, S_T, workspace)
    shape = _shape_of(q, v, gate_f, cu_seqlens, chunk, validate, recurrent, state_ctas, grid_ctas)
    shape.flags |= _GATE_MODES[gate_mode]
    N = shape.B if cu_seqlens is None else shape.n_seqs
    if o is None:
        o = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    if S_T is None and output_final_state:
        S_T = torch.empty((N, shape.H, shape.dk, shape.dv), dtype=torch.float32, device=q.device)
    need = kda_chunk_fwd_workspace_size(shape)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load_library().kda_chunk_fwd_layer(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(gate_f), _ptr(A_log), _ptr(dt_bias), _ptr(beta),
        _ptr(S0), _ptr(cu_seqlens), _ptr(out_gate), _ptr(norm_weight), float(eps), _ptr(o), _ptr(S_T),
        _ptr(workspace), ws_bytes, _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd_layer")
    return o, S_T


def kda_decode_step_layer(q, k, v, gate_f, A_log, dt_bias, beta, state, *, state_slots=None, out_gate=None,
                          norm_weight=None, eps: float = 1e-5, o=None, stream=None):
    """One decode step with the layer's producer steps (raw q, k; decay gate
    from gate_f, A_log, dt_bias) and the optional output epilogue; ``state``
    is updated in place (dense rows, or pool slots with ``state_slots``).
    Inputs [N, H, d] (one token per sequence) or [N, 1, H, d]; returns o."""
    import torch
    if q.dim() == 3:
        q, k, v, gate_f = (t.unsqueeze(1) for t in (q, k, v, gate_f))
        beta = beta.unsqueeze(1)
        if out_gate is not None:
            out_gate = out_gate.unsqueeze(1)
    N, _, H, dk = q.shape
    if (out_gate is None) != (norm_weight is None):
        raise ValueError("out_gate and norm_weight go together")
    if A_log.dtype != torch.float32 or dt_bias.dtype != torch.float32:
        raise ValueError("A_log and dt_bias must be float32")
    if A_log.numel() != H or dt_bias.numel() != H * dk:
        raise ValueError("A_log must have H values and dt_bias H * dk")
    _need_cuda(q, k, v, gate_f, A_log, dt_bias, beta, state, state_slots, out_gate, norm_weight, o)
    shape = _shape_of(q, v, gate_f, None, 64, False)
    if o is None:
        o = torch.empty((N, H, v.shape[-1]), dtype=v.dtype, device=v.device)
    num_slots = 0
    if state_slots is not None:
        _check_slots(state, state_slots, N)
        num_slots = state.shape[0]
    rc = load_library().kda_decode_step_layer(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(gate_f), _ptr(A_log), _ptr(dt_bias), _ptr(beta),
        _ptr(state), _ptr(state_slots), num_slots, _ptr(out_gate), _ptr(norm_weight), float(eps), _ptr(o),
        _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_decode_step_layer")
    return o


class PrefillPlanInfo(ctypes.Structure):
    """kda_prefill_plan_info (include/kda.h)."""
    _fields_ = [("state_ctas", ctypes.c_int32), ("grid_ctas", ctypes.c_int32), ("ring_depth", ctypes.c_int32),
                ("fuse_output_gate", ctypes.c_int32), ("workspace_bytes", ctypes.c_uint64),
                ("min_workspace_bytes", ctypes.c_uint64)]


def kda_prefill_plan(shape, num_sms: int = 0) -> dict:
    """The tensor-core prefill's plan for ``shape`` (a kda_shape) on a device
    with ``num_sms`` SMs (0: the current device): state / transform CTA split,
    ring depth, output-epilogue placement and workspace sizes."""
    info = PrefillPlanInfo()
    rc = load_library().kda_prefill_plan(ctypes.byref(shape), int(num_sms), ctypes.byref(info))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_prefill_plan")
    return {name: getattr(info, name) for name, _ in PrefillPlanInfo._fields_}


def kda_chunk_fwd_noalloc(q, k, v, log_alpha, beta, S0, cu_seqlens, o, S_T, *, chunk: int = 64, stream=None,
                          state_ctas: int = 0, grid_ctas: int = 0):
    """kda_chunk_fwd on the library's built-in scratch array (no workspace).

    For callers that cannot allocate device memory where they run the prefill
    (see include/kda.h for the size limit and the sharing rules).  o and S_T
    are caller-owned outputs; nothing is allocated here.
    """
    _need_cuda(q, k, v, log_alpha, beta, S0, cu_seqlens, o, S_T)
    shape = _shape_of(q, v, log_alpha, cu_seqlens, chunk, False, False, state_ctas, grid_ctas)
    rc = load_library().kda_chunk_fwd_noalloc(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0),
        _ptr(cu_seqlens), _ptr(o), _ptr(S_T), _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd_noalloc")
    return o, S_T


def _check_slots(state_pool, state_slots, n, has_initial_state=None):
    import torch
    if state_pool.dtype != torch.float32 or state_pool.dim() != 4:
        raise ValueError("state_pool must be a [num_slots, H, dk, dv] float32 tensor")
    if state_slots.dtype != torch.int32 or state_slots.numel() != n:
        raise ValueError(f"state_slots must be an int32 tensor with one entry per sequence ({n})")
    if has_initial_state is not None and (has_initial_state.dtype not in (torch.uint8, torch.bool)
                                          or has_initial_state.numel() != n):
        raise ValueError(f"has_initial_state must be a uint8/bool tensor with one entry per sequence ({n})")


def kda_chunk_fwd_slots(q, k, v, log_alpha, beta, state_pool, state_slots, has_initial_state=None,
                        cu_seqlens=None, *, chunk: int = 64, o=None, workspace=None, stream=None,
                        validate: bool = False, recurrent: bool = False, state_ctas: int = 0,
                        grid_ctas: int = 0):
    """Prefill on a slot-indexed state pool (include/kda.h, serving-state
    variants).  Sequence n starts from ``state_pool[state_slots[n]]`` (or from
    zeros where ``has_initial_state[n]`` is 0) and its final state is written
    back there; a negative slot is padding (zero start, state dropped).
    Returns o."""
    import torch
    _need_cuda(q, k, v, log_alpha, beta, state_pool, state_slots, has_initial_state, cu_seqlens, o, workspace)
    shape = _shape_of(q, v, log_alpha, cu_seqlens, chunk, validate, recurrent, state_ctas, grid_ctas)
    N = shape.B if cu_seqlens is None else shape.n_seqs
    _check_slots(state_pool, state_slots, N, has_initial_state)
    if o is None:
        o = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    need = kda_chunk_fwd_workspace_size(shape)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load_library().kda_chunk_fwd_slots(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(state_pool),
        int(state_pool.shape[0]), _ptr(state_slots), _ptr(has_initial_state), _ptr(cu_seqlens), _ptr(o),
        _ptr(workspace), ws_bytes, _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd_slots")
    return o


def kda_decode_step_slots(q, k, v, log_alpha, beta, state_pool, state_slots, *, o=None, stream=None):
    """One recurrent token per row on a slot-indexed state pool: row n updates
    ``state_pool[state_slots[n]]`` in place (negative slot: padding, zero
    state, nothing written).  Returns o [N,H,dv]."""
    import torch
    _need_cuda(q, k, v, log_alpha, beta, state_pool, state_slots, o)
    N, H, dk = q.shape
    dv = v.shape[-1]
    _check_slots(state_pool, state_slots, N)
    shape = make_shape(N, 1, H, dk, dv, 64, 0, _dtype_code(q), _dtype_code(log_alpha), 0)
    if o is None:
        o = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    rc = load_library().kda_decode_step_slots(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(state_pool),
        int(state_pool.shape[0]), _ptr(state_slots), _ptr(o), _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_decode_step_slots")
    return o


def kda_decode_step(q, k, v, log_alpha, beta, S, *, o=None, stream=None):
    """One recurrent token: q, k, log_alpha [N,H,dk]; v [N,H,dv]; beta [N,H];
    S [N,H,dk,dv] fp32 updated in place.  Returns o [N,H,dv]."""
    import torch
    _need_cuda(q, k, v, log_alpha, beta, S, o)
    N, H, dk = q.shape
    dv = v.shape[-1]
    shape = make_shape(N, 1, H, dk, dv, 64, 0, _dtype_code(q), _dtype_code(log_alpha), 0)
    if o is None:
        o = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    rc = load_library().kda_decode_step(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                        _ptr(beta), _ptr(S), _ptr(o), _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_decode_step")
    return o


def kda_check_device_error(stream=None) -> int:
    """Synchronise and return (and clear) the device-side error code."""
    return int(load_library().kda_check_device_error(_stream(stream)))
