"""The checked build (MSS_DEBUG=1, libsss48_debug.so) on the GPU.

The checked build bounds-checks every global access at a computed index
and reports one outside its tensor through the status calls, without
trapping.  Here: it computes the same results as the ordinary build and
reports no error on valid calls (forward scan, split and unsplit, the
plain-load path, decode and backward), and a planted out-of-range store
(test flag, checked build only) is skipped and reported as
MSS_ERR_INVALID_ARG.  The planted index lands inside padding allocated
after y, so the test stays in bounds even if the check were missing.
"""
import ctypes

import pytest
import torch

import selective_state_space_48_b200 as sss
import workloads
from scan_checks import gpu_inputs, norm_err, run_oracle, tolerance

pytestmark = pytest.mark.gpu


def _scan(lib, w, inp, y, plan_splits=0, test_flags=0):
    args = sss.make_scan_args(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                              z=inp["z"], delta_bias=inp["delta_bias"], y=y,
                              plan_splits=plan_splits, test_flags=test_flags)
    ws = sss.alloc_workspace(sss.scan_workspace_size(args), y.device)
    if ws is not None:
        args.workspace, args.workspace_bytes = ws.data_ptr(), ws.numel()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.mamba_selective_scan_fwd(ctypes.byref(args), stream) == sss.MSS_OK
    rc = lib.mss_scan_status(ctypes.byref(args), stream)
    return rc, ws


@pytest.mark.parametrize("L,splits,dt", [(1000, 0, "bf16"), (4096, 4, "f32"), (301, 0, "f32")])
def test_checked_build_matches_and_reports_nothing(L, splits, dt):
    dbg = sss.load_debug_library()
    w = workloads.custom(2, 40, 16, L, in_dtype=dt, has_z=True)
    inp = gpu_inputs(w, seed=61 + L)
    y = torch.empty(w.batch, w.dim, w.seqlen, device="cuda")
    rc, _ = _scan(dbg, w, inp, y, plan_splits=splits)
    assert rc == sss.MSS_OK
    assert norm_err(y.cpu(), run_oracle(w, inp)) <= tolerance(dt)


def test_planted_out_of_range_store_is_skipped_and_reported():
    dbg = sss.load_debug_library()
    w = workloads.custom(1, 32, 16, 64, in_dtype="f32", has_z=True)
    inp = gpu_inputs(w, seed=62)
    n = w.batch * w.dim * w.seqlen
    buf = torch.full((2 * n + 64,), 12345.0, device="cuda")
    y = buf[:n].view(w.batch, w.dim, w.seqlen)
    rc, _ = _scan(dbg, w, inp, y, test_flags=sss.MSS_TESTFLAG_DEBUG_OOB)
    torch.cuda.synchronize()
    assert rc == sss.MSS_ERR_INVALID_ARG
    # nothing was written past y
    assert torch.all(buf[n:] == 12345.0)
    # the skipped store is channel 0, steps 0..3; every other output is right
    want = run_oracle(w, inp)
    got = y.cpu().numpy()
    assert (got[0, 0, :4] == 12345.0).all()
    got[0, 0, :4] = want[0, 0, :4]
    assert norm_err(got, want) <= tolerance("f32")
    # the word was cleared by the read: a clean call reports OK
    y2 = torch.empty_like(y)
    rc, _ = _scan(dbg, w, inp, y2)
    assert rc == sss.MSS_OK


def test_ordinary_build_ignores_the_checked_build_flag():
    lib = sss.load_library()
    w = workloads.custom(1, 32, 16, 64, in_dtype="f32", has_z=True)
    inp = gpu_inputs(w, seed=62)
    y = torch.empty(w.batch, w.dim, w.seqlen, device="cuda")
    rc, _ = _scan(lib, w, inp, y, test_flags=sss.MSS_TESTFLAG_DEBUG_OOB)
    assert rc == sss.MSS_OK
    assert norm_err(y.cpu(), run_oracle(w, inp)) <= tolerance("f32")


def test_checked_build_decode_and_backward():
    dbg = sss.load_debug_library()
    # decode through the checked library
    batch, dim, N = 3, 70, 16
    g = torch.Generator(device="cuda")
    g.manual_seed(63)
    r = lambda *s: torch.randn(*s, generator=g, device="cuda")
    state, x, dtv = r(batch, dim, N), r(batch, dim), r(batch, dim)
    A = -torch.rand(dim, N, generator=g, device="cuda") * 3
    B, C = r(batch, N), r(batch, N)
    y = torch.empty(batch, dim, device="cuda")
    st1, st2 = state.clone(), state.clone()
    a = sss.UpdateArgs()
    a.batch, a.dim, a.dstate = batch, dim, N
    a.in_dtype = a.out_dtype = sss.MSS_F32
    a.state, a.x, a.dt, a.A, a.B, a.C = (t.data_ptr() for t in (st1, x, dtv, A, B, C))
    a.dt_softplus, a.y = 1, y.data_ptr()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert dbg.selective_state_update(ctypes.byref(a), stream) == sss.MSS_OK
    want = sss.selective_state_update(st2, x, dtv, A, B, C)
    torch.cuda.synchronize()
    assert torch.equal(y, want) and torch.equal(st1, st2)
    # backward through the checked library: same gradients as the ordinary one
    w = workloads.custom(1, 48, 16, 200, in_dtype="bf16", has_z=True)
    inp = gpu_inputs(w, seed=64)
    dy = torch.randn(1, 48, 200, generator=g, device="cuda")
    ref = sss.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy,
                                 D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"])
    ba = sss.ScanBwdArgs()
    ba.batch, ba.dim, ba.dstate, ba.seqlen = w.batch, w.dim, w.dstate, w.seqlen
    ba.in_dtype = sss.MSS_BF16
    ptr = lambda t: None if t is None else t.data_ptr()
    for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias"):
        setattr(ba, k, ptr(inp[k]))
    ba.delta_softplus = 1
    ba.dy = dy.data_ptr()
    out = {k: torch.empty_like(v) for k, v in ref.items() if v is not None}
    for k, v in out.items():
        setattr(ba, k, v.data_ptr())
    nb = ctypes.c_size_t(0)
    assert dbg.mss_scan_bwd_workspace_size(ctypes.byref(ba), ctypes.byref(nb)) == sss.MSS_OK
    ws = torch.empty(int(nb.value), dtype=torch.uint8, device="cuda")
    ba.workspace, ba.workspace_bytes = ws.data_ptr(), int(nb.value)
    assert dbg.mamba_selective_scan_bwd(ctypes.byref(ba), stream) == sss.MSS_OK
    torch.cuda.synchronize()
    for k, v in out.items():
        assert norm_err(v.cpu(), ref[k].cpu()) <= 1e-5, k
    # nothing was recorded in the library's word by the decode or backward
    args = sss.make_scan_args(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                              y=torch.empty(1, 48, 200, device="cuda"))
    assert dbg.mss_scan_status(ctypes.byref(args), stream) == sss.MSS_OK
