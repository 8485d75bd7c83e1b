"""Failure detection: a device-side bounded wait runs out, the call reports
KDA_ERR_TIMEOUT, and the GPU stays usable.

Every wait in the library's kernels is bounded; one that gives up records
KDA_ERR_TIMEOUT in the library's device error word and raises an abort flag
that every CTA polls, so the launch ends and the error surfaces through
kda_check_device_error().  The test runs the test-only build
(libkda_testhooks.so, compiled with -DKDA_TEST_HOOKS): its waits give up after
~0.1 s instead of ~2 s, and a host-armed flag makes one state CTA skip the
signal that its first U^T product is complete -- a wait that nothing will
end.  No fault, trap or endless loop is involved: the missing signal is the
only change, and the kernel must unwind by itself.  A following call with the
flag disarmed must then match the fp64 oracle.
"""
import ctypes

import numpy as np
import pytest
import torch

import gated_delta_rule_110_b200 as kda
import oracle
from gated_delta_rule_110_b200 import build as kbuild
from gated_delta_rule_110_b200 import inputs as gen
from tests.conftest import max_rel_l2_per_slice

pytestmark = pytest.mark.gpu


def _hooks_lib():
    lib = ctypes.CDLL(str(kbuild.TEST_LIB))
    vp, sp = ctypes.c_void_p, ctypes.POINTER(kda.kda_shape)
    lib.kda_chunk_fwd_workspace_size.argtypes = [sp]
    lib.kda_chunk_fwd_workspace_size.restype = ctypes.c_size_t
    lib.kda_chunk_fwd.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.kda_chunk_fwd.restype = ctypes.c_int
    lib.kda_check_device_error.argtypes = [vp]
    lib.kda_check_device_error.restype = ctypes.c_int
    lib.kda_test_set_skip_commit.argtypes = [ctypes.c_int]
    lib.kda_test_set_skip_commit.restype = ctypes.c_int
    return lib


def test_bounded_wait_times_out_and_the_gpu_recovers():
    lib = _hooks_lib()
    x = gen.make_inputs(1, 256, 2, 128, 128, seed=41)
    xd = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    shape = kda.make_shape(1, 256, 2, 128, 128, 64, 0, kda.KDA_BF16, kda.KDA_BF16)
    ws = torch.empty(lib.kda_chunk_fwd_workspace_size(ctypes.byref(shape)), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(xd["v"])
    S = torch.empty_like(xd["S0"])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())

    def call():
        return lib.kda_chunk_fwd(ctypes.byref(shape), p(xd["q"]), p(xd["k"]), p(xd["v"]), p(xd["log_alpha"]),
                                 p(xd["beta"]), p(xd["S0"]), None, p(o), p(S), p(ws), ws.numel(), stream)

    assert lib.kda_test_set_skip_commit(1) == 0
    try:
        assert call() == 0                                   # the launch itself succeeds
        assert lib.kda_check_device_error(stream) == -8      # KDA_ERR_TIMEOUT, reported on the host
        assert lib.kda_check_device_error(stream) == 0       # ... and cleared
    finally:
        assert lib.kda_test_set_skip_commit(0) == 0
    # the context is intact: the same call now runs to completion and is correct
    assert call() == 0
    assert lib.kda_check_device_error(stream) == 0
    o_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"])
    assert max_rel_l2_per_slice(o.float().cpu().numpy(), o_ref, (0, 2)) <= 2e-2
    assert max_rel_l2_per_slice(S.cpu().numpy(), S_ref, (0, 1)) <= 2e-2
    assert np.isfinite(o.float().cpu().numpy()).all()
