"""The allocation-free scan entry point (needs a GPU).

Some callers cannot allocate device memory (plugins handed only their own
tensors, code under a pool it must not re-enter, paths where cudaMalloc may
not run).  mamba_selective_scan_fwd_noalloc serves them from a fixed array
the library owns.  This file is collected last so a stop-at-first-failure
run has already run every other test; it also passes alone in a fresh
process.
"""
import ctypes

import pytest
import torch

import selective_state_space_48_b200 as sss
import workloads
from scan_checks import gpu_inputs, norm_err, tolerance

pytestmark = pytest.mark.gpu


def _call_noalloc(args):
    lib = sss.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.mamba_selective_scan_fwd_noalloc(ctypes.byref(args), stream)


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_noalloc_matches_the_workspace_entry_point(dt):
    # few channels and a long sequence: the plan splits the sequence, so the
    # scan needs scratch memory
    w = workloads.custom(1, 64, 16, 40000, in_dtype=dt, has_z=True)
    inp = gpu_inputs(w, seed=31, h0=True)
    want, want_last = sss.selective_scan_fwd(
        inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
        z=inp["z"], delta_bias=inp["delta_bias"], h0=inp["h0"],
        return_last_state=True, check_status=True)
    y = torch.empty_like(want)
    last = torch.empty_like(want_last)
    args = sss.make_scan_args(inp["u"], inp["delta"], inp["A"], inp["B"],
                              inp["C"], D=inp["D"], z=inp["z"],
                              delta_bias=inp["delta_bias"], h0=inp["h0"],
                              y=y, last_state=last)
    assert sss.scan_workspace_size(args) > 0
    tol = tolerance(dt)
    for call in range(2):
        y.fill_(float("nan"))
        last.fill_(float("nan"))
        assert _call_noalloc(args) == sss.MSS_OK
        torch.cuda.synchronize()
        assert norm_err(y.cpu(), want.cpu()) <= tol, call
        assert norm_err(last.cpu(), want_last.cpu()) <= tol, call


def test_noalloc_without_split_matches():
    w = workloads.custom(2, 96, 16, 300, in_dtype="bf16", has_z=True)
    inp = gpu_inputs(w, seed=32)
    want = sss.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"],
                                  inp["C"], D=inp["D"], z=inp["z"],
                                  delta_bias=inp["delta_bias"])
    y = torch.empty_like(want)
    args = sss.make_scan_args(inp["u"], inp["delta"], inp["A"], inp["B"],
                              inp["C"], D=inp["D"], z=inp["z"],
                              delta_bias=inp["delta_bias"], y=y)
    for _ in range(2):
        y.zero_()
        assert _call_noalloc(args) == sss.MSS_OK
        torch.cuda.synchronize()
        assert norm_err(y.cpu(), want.cpu()) <= tolerance("bf16")


def test_noalloc_rejects_plans_beyond_its_array():
    a = sss.ScanArgs()
    # 128 channel tiles x 64 chunks need far more than the 8 MiB array
    a.batch, a.dim, a.dstate, a.seqlen = 1, 4096, 16, 65536
    a.in_dtype, a.out_dtype = sss.MSS_BF16, sss.MSS_F32
    a.u = a.delta = a.A = a.B = a.C = a.y = 0x10000
    a.plan_splits = 64
    assert sss.scan_workspace_size(a) > (8 << 20)
    assert _call_noalloc(a) == sss.MSS_ERR_WORKSPACE


def _noalloc_status(args):
    lib = sss.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.mss_scan_noalloc_status(ctypes.byref(args), stream)


def test_noalloc_reports_a_timed_out_wait_and_recovers():
    """A publication that never comes (test flag): the bounded wait before
    the chunks' carries are composed runs out, mss_scan_noalloc_status
    reports it from the word in the library's array, and the next call is
    correct and reports OK."""
    w = workloads.custom(1, 32, 16, 4096, in_dtype="f32", has_z=False)
    inp = gpu_inputs(w, seed=2)
    want = sss.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"],
                                  inp["C"], D=inp["D"], delta_bias=inp["delta_bias"],
                                  plan_splits=4, check_status=True)
    y = torch.empty_like(want)
    bad = sss.make_scan_args(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                             D=inp["D"], delta_bias=inp["delta_bias"], y=y,
                             plan_splits=4, test_flags=sss.MSS_TESTFLAG_DROP_PUBLISH,
                             spin_timeout_ns=20_000_000)
    assert sss.scan_workspace_size(bad) > 0
    assert _call_noalloc(bad) == sss.MSS_OK
    assert _noalloc_status(bad) == sss.MSS_ERR_TIMEOUT
    # the word was read and cleared
    assert _noalloc_status(bad) == sss.MSS_OK
    good = sss.make_scan_args(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                              D=inp["D"], delta_bias=inp["delta_bias"], y=y,
                              plan_splits=4)
    assert _call_noalloc(good) == sss.MSS_OK
    assert _noalloc_status(good) == sss.MSS_OK
    assert norm_err(y.cpu(), want.cpu()) <= tolerance("f32")
