"""lr_rglru_fwd_noalloc: the rglru forward pass for callers that cannot allocate device memory
(a host framework that owns every device byte and hands plug-ins no scratch, a fixed plug-in
callback, or a latency-critical loop where cudaMalloc would synchronise the device).  Its scratch
is a fixed array inside the library, so the caller passes only inputs and outputs.

This file is collected last on purpose: if it fails, a run that stops at the first failure has
already run every other test.  It checks, through the C ABI, that two calls in a row (the second
one on different inputs, so stale scratch contents would show) give the same y and checkpoints
as lr_scan_fwd with a caller-provided workspace, within the fp32 tolerance of the other parity
tests, and that problems too large for the array are rejected before any GPU work.
"""
import ctypes

import pytest
import torch

from helpers import assert_close
from selective_state_space_09_b200 import inputs

pytestmark = pytest.mark.gpu


def _noalloc(lrscan):
    f = lrscan.lib.lr_rglru_fwd_noalloc
    f.argtypes = [ctypes.POINTER(lrscan.Desc), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    f.restype = ctypes.c_int
    return f


def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    from selective_state_space_09_b200 import lrscan
    f = _noalloc(lrscan)
    w = inputs.WORKLOADS["rglru"]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, seed in enumerate((11, 12)):
        inp = {k: v.cuda() for k, v in inputs.rglru(w["B"], w["L"], w["D"], seed=seed).items()}
        plan = lrscan.plan_for("rglru", {"a": inp["a"], "b": inp["b"]}, w["segment"])
        y_ref = torch.empty_like(inp["b"])
        plan.fwd({"a": inp["a"], "b": inp["b"]}, y_ref)
        ck_ref = plan.ckpt_view().clone()

        y = torch.full_like(inp["b"], float("nan"))
        ck = torch.full((lrscan.ckpt_bytes(plan.desc) // 4,), float("nan"), device="cuda")
        s = f(ctypes.byref(plan.desc), inp["a"].data_ptr(), inp["b"].data_ptr(), y.data_ptr(),
              ck.data_ptr(), stream, 1 if call == 1 else 0)
        torch.cuda.synchronize()
        assert s == 0, lrscan.lib.lr_status_string(s)
        assert_close("y (call %d)" % call, y, y_ref.cpu().double().numpy(), 1e-5)
        assert_close("ckpt (call %d)" % call, ck.view(ck_ref.shape), ck_ref.cpu().double().numpy(), 1e-5)


def test_noalloc_rejects_problems_beyond_its_scratch():
    from selective_state_space_09_b200 import lrscan
    f = _noalloc(lrscan)
    big = lrscan.make_desc("rglru", torch.float32, B=64, L=4096, D=4096, segment=128)
    p = ctypes.c_void_p(256)  # never dereferenced: the size check comes first
    assert f(ctypes.byref(big), p, p, p, p, None, 0) == 4          # LR_ERR_WORKSPACE
    other = lrscan.make_desc("rotlru", torch.float32, B=1, L=64, D=64, segment=64)
    assert f(ctypes.byref(other), p, p, p, p, None, 0) == 1        # not the rglru kind


def test_noalloc_reports_a_bounded_wait_that_gave_up():
    """The failure path through the library's array: with the test hook that makes the first
    segment's tiles withhold their carry, the tiles of the later segments wait out their 1 s bound
    and record LR_ERR_TIMEOUT.  check = 1 returns it; with check = 0 the error query reads it, and
    the next call (without the hook) clears it and succeeds."""
    from selective_state_space_09_b200 import lrscan
    f = _noalloc(lrscan)
    q = lrscan.lib.lr_rglru_noalloc_error
    q.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32)]
    q.restype = ctypes.c_int
    inp = {k: v.cuda() for k, v in inputs.rglru(1, 512, 64, seed=21).items()}
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    desc = lrscan.make_desc("rglru", torch.float32, B=1, L=512, D=64, segment=128)
    desc.flags |= lrscan.TEST_WITHHOLD_CARRY
    y = torch.empty_like(inp["b"])
    ck = torch.empty((lrscan.ckpt_bytes(desc) // 4,), device="cuda")
    args = (inp["a"].data_ptr(), inp["b"].data_ptr(), y.data_ptr(), ck.data_ptr(), stream)
    assert f(ctypes.byref(desc), *args, 1) == 6                      # LR_ERR_TIMEOUT
    assert f(ctypes.byref(desc), *args, 0) == 0                      # enqueued
    info = ctypes.c_int32(0)
    assert q(stream, ctypes.byref(info)) == 6                        # read ...
    assert q(stream, ctypes.byref(info)) == 0                        # ... and cleared
    desc.flags &= ~lrscan.TEST_WITHHOLD_CARRY
    assert f(ctypes.byref(desc), *args, 1) == 0                      # the context is still usable
    ref = lrscan.plan_for("rglru", {"a": inp["a"], "b": inp["b"]}, 128)
    y_ref = torch.empty_like(y)
    ref.fwd({"a": inp["a"], "b": inp["b"]}, y_ref)
    torch.cuda.synchronize()
    assert_close("y after the timeout", y, y_ref.cpu().double().numpy(), 1e-5)
