"""Backward scan against the fp64 oracle backward (needs a GPU).

The oracle's gradients are pinned by central finite differences of the
forward oracle on the CPU.  Here every gradient of the CUDA backward (du,
ddelta, dA, dB, dC, dD, dz, ddelta_bias, dh0) is compared with the oracle on
the same inputs (bf16 cases: the oracle reads the same bf16-rounded values),
as max |g_gpu - g_ref| / max |g_ref| per tensor.  Both sides do the same
arithmetic; the GPU does it in fp32 with atomic sums over channels and
batch rows, hence the fp32-level bound.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import selective_state_space_48_b200 as sss
import workloads
from oracle.compare import ErrorStats
from scan_checks import gpu_inputs, norm_err

pytestmark = pytest.mark.gpu

TOL = 1e-4

NAMES = ("du", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias", "dh0")


def _grads(w, inp, dy, d_last, softplus=True):
    g_gpu = sss.selective_scan_bwd(
        inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy, D=inp["D"],
        z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=softplus,
        h0=inp["h0"], d_last=d_last)
    torch.cuda.synchronize()
    h = workloads.to_numpy_f64(inp)
    g_ref = oracle.selective_scan_bwd(
        h["u"], h["delta"], h["A"], h["B"], h["C"], dy.double().cpu().numpy(),
        D=h["D"], z=h["z"], delta_bias=h["delta_bias"], delta_softplus=softplus,
        h0=h["h0"], d_last=None if d_last is None else d_last.double().cpu().numpy())
    return g_gpu, g_ref


def _compare(g_gpu, g_ref, what):
    errs = {}
    for k in NAMES:
        if g_ref.get(k) is None:
            assert g_gpu.get(k) is None, (what, k)
            continue
        errs[k] = norm_err(g_gpu[k].cpu().numpy(), g_ref[k])
    bad = {k: e for k, e in errs.items() if not e <= TOL}
    assert not bad, (what, bad, errs)


CASES = [
    # name, batch, dim, N, L, dtype
    ("f32-ragged", 2, 40, 16, 300, "f32"),
    ("f32-N5", 1, 64, 5, 333, "f32"),
    ("f32-N4-tiny", 1, 32, 4, 17, "f32"),
    ("bf16", 2, 48, 16, 1000, "bf16"),
    ("bf16-N12", 1, 33, 12, 129, "bf16"),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_the_oracle(case):
    name, batch, dim, N, L, dt = case
    w = workloads.custom(batch, dim, N, L, in_dtype=dt, has_z=True, a_noise=0.1)
    inp = gpu_inputs(w, seed=5000 + len(name), h0=True)
    g = torch.Generator(device="cuda")
    g.manual_seed(5100 + len(name))
    dy = torch.randn(batch, dim, L, generator=g, device="cuda")
    d_last = torch.randn(batch, dim, N, generator=g, device="cuda")
    _compare(*_grads(w, inp, dy, d_last), name)


def test_backward_without_optional_inputs_and_softplus_off():
    w = workloads.custom(2, 40, 16, 200, in_dtype="f32", has_z=False,
                         has_delta_bias=False, has_D=False, softplus=False)
    inp = gpu_inputs(w, seed=5200, h0=False)
    inp["delta"] = inp["delta"].abs() * 0.1 + 0.01  # positive steps without softplus
    dy = torch.randn(2, 40, 200, device="cuda")
    _compare(*_grads(w, inp, dy, None, softplus=False), "no optional inputs")


def test_backward_of_the_last_state_alone():
    """dy = 0: every gradient flows from d_last through the recurrence."""
    w = workloads.custom(1, 32, 16, 160, in_dtype="f32", has_z=True)
    inp = gpu_inputs(w, seed=5201, h0=True)
    dy = torch.zeros(1, 32, 160, device="cuda")
    d_last = torch.randn(1, 32, 16, device="cuda")
    _compare(*_grads(w, inp, dy, d_last), "last state only")


def _full_tolerance(terms: int) -> float:
    """Bound for a gradient that the GPU accumulates as an fp32 sum of
    `terms` contributions (atomics over channels or over (batch row, step)):
    recursive summation errs by at most (terms - 1) u of the sum of the
    magnitudes (u = 2^-24), on top of the fp32 recurrence's own 1e-4."""
    return TOL + terms * 2.0 ** -24


def test_backward_at_the_130m_layer_shape_every_element():
    """The backward at the shape `bench.py --pass bwd` times (Mamba-130M
    layer: batch 8, D 1536, N 16, L 2048, bf16 inputs): every element of
    all gradients against the oracle backward, run one batch row at a time
    (dA, dD, ddelta_bias summed over the rows in fp64)."""
    w = workloads.BY_NAME["mamba130m-layer"]
    inp = gpu_inputs(w)
    g = torch.Generator(device="cuda")
    g.manual_seed(48000)
    dy = torch.randn(w.batch, w.dim, w.seqlen, generator=g, device="cuda")
    got = sss.selective_scan_bwd(
        inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy, D=inp["D"],
        z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=w.softplus)
    torch.cuda.synchronize()
    host = lambda t, b: None if t is None else t[b:b + 1].detach().float().cpu().double().numpy()
    par = lambda t: None if t is None else t.detach().float().cpu().double().numpy()
    sums = {"dA": 0.0, "dD": 0.0, "ddelta_bias": 0.0}
    stats = {k: ErrorStats() for k in ("du", "ddelta", "dz", "dB", "dC")}
    for b in range(w.batch):
        ref = oracle.selective_scan_bwd(
            host(inp["u"], b), host(inp["delta"], b), par(inp["A"]), host(inp["B"], b),
            host(inp["C"], b), host(dy, b), D=par(inp["D"]), z=host(inp["z"], b),
            delta_bias=par(inp["delta_bias"]), delta_softplus=w.softplus)
        for k in stats:
            stats[k].add(got[k][b:b + 1].cpu().numpy(), ref[k])
        for k in sums:
            sums[k] = sums[k] + ref[k]
    errs = {k: st.norm_err for k, st in stats.items()}
    for k, ref in sums.items():
        errs[k] = norm_err(got[k].cpu().numpy(), ref)
    bound = {"du": TOL, "ddelta": TOL, "dz": TOL,
             "dB": _full_tolerance(w.dim), "dC": _full_tolerance(w.dim),
             "dA": _full_tolerance(w.batch * w.seqlen),
             "dD": _full_tolerance(w.batch * w.seqlen),
             "ddelta_bias": _full_tolerance(w.batch * w.seqlen)}
    bad = {k: (e, bound[k]) for k, e in errs.items() if not e <= bound[k]}
    assert not bad, (bad, errs)


@pytest.mark.parametrize("dt,L", [("bf16", 1024), ("bf16", 777), ("f32", 512)])
def test_backward_reads_strided_views(dt, L):
    """u and z as the two halves of one (batch, 2 D, L) projection, B and C
    as rows of one (batch, 2 N + 3, L) tensor and dy as a slice of a wider
    one, read in place: every gradient matches the oracle, and the same
    backward of packed copies.  L = 1024 stages whole aligned rows with
    16-byte copies through the strides; L = 777 and fp32 take element
    loads for the rows that are not whole 16-byte pieces."""
    batch, D, N = 2, 72, 16
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    w = workloads.custom(batch, D, N, L, in_dtype=dt, has_z=True, a_noise=0.1)
    inp = gpu_inputs(w, seed=4242 + L, h0=True)
    proj = torch.empty(batch, 2 * D, L, dtype=tdt, device="cuda")
    proj[:, :D], proj[:, D:] = inp["u"], inp["z"]
    xb = torch.zeros(batch, 2 * N + 3, L, dtype=tdt, device="cuda")
    xb[:, 1:N + 1], xb[:, N + 2:2 * N + 2] = inp["B"], inp["C"]
    g = torch.Generator(device="cuda")
    g.manual_seed(4343)
    wide = torch.randn(batch, D + 5, L, generator=g, device="cuda")
    dy = wide[:, 3:D + 3]
    views = dict(inp, u=proj[:, :D], z=proj[:, D:], B=xb[:, 1:N + 1], C=xb[:, N + 2:2 * N + 2])
    assert not views["u"].is_contiguous() and not dy.is_contiguous()
    g_view, g_ref = _grads(w, views, dy, None)
    _compare(g_view, g_ref, f"strided {dt} L={L}")
    g_pack = sss.selective_scan_bwd(
        inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy.contiguous(), D=inp["D"],
        z=inp["z"], delta_bias=inp["delta_bias"], h0=inp["h0"])
    for k in NAMES:
        if g_pack.get(k) is None:
            continue
        assert norm_err(g_view[k].cpu().numpy(), g_pack[k].cpu().numpy()) <= 1e-6, k


PACKED = [
    # name, batch, dim, N, L, dtype, interior starts
    ("f32-blocks", 2, 40, 16, 300, "f32", [1, 16, 17, 150, 151, 299]),
    ("bf16-long", 1, 48, 16, 1000, "bf16", [5, 32, 33, 500, 999]),
    ("f32-N5", 1, 33, 5, 77, "f32", [2, 3, 40]),
]


@pytest.mark.parametrize("case", PACKED, ids=[c[0] for c in PACKED])
def test_backward_packed_sequences(case):
    """Packed sequences (starts on and next to 16-step block boundaries, at
    step 1 and at the last step, one-step sequences): every gradient against
    the oracle backward with the same packing, where nothing flows across a
    sequence start."""
    name, batch, dim, N, L, dt, starts = case
    w = workloads.custom(batch, dim, N, L, in_dtype=dt, has_z=True, a_noise=0.1)
    inp = gpu_inputs(w, seed=5150 + L, h0=True)
    cu = sorted(set([0, L] + starts))
    cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(5151 + L)
    dy = torch.randn(batch, dim, L, generator=g, device="cuda")
    d_last = torch.randn(batch, dim, N, generator=g, device="cuda")
    g_gpu = sss.selective_scan_bwd(
        inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy, D=inp["D"],
        z=inp["z"], delta_bias=inp["delta_bias"], h0=inp["h0"], d_last=d_last,
        cu_seqlens=cu_t)
    torch.cuda.synchronize()
    h = workloads.to_numpy_f64(inp)
    g_ref = oracle.selective_scan_bwd(
        h["u"], h["delta"], h["A"], h["B"], h["C"], dy.double().cpu().numpy(),
        D=h["D"], z=h["z"], delta_bias=h["delta_bias"], h0=h["h0"],
        d_last=d_last.double().cpu().numpy(), cu_seqlens=cu)
    _compare(g_gpu, g_ref, name)


def test_packed_backward_rejects_checkpoints():
    w = workloads.custom(1, 32, 16, 64, in_dtype="f32", has_z=False)
    inp = gpu_inputs(w, seed=5)
    cu_t = torch.tensor([0, 10, 64], dtype=torch.int32, device="cuda")
    ck = sss.scan_checkpoints(1, 32, 16, 64, "cuda")
    dy = torch.ones(1, 32, 64, device="cuda")
    with pytest.raises(sss.MssError) as ei:
        sss.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy,
                               cu_seqlens=cu_t, checkpoints=ck)
    assert ei.value.code == sss.MSS_ERR_UNSUPPORTED


def _bwd_ws(inp, dy, d_last, workspace, checkpoints=None):
    g = sss.selective_scan_bwd(
        inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy, D=inp["D"],
        z=inp["z"], delta_bias=inp["delta_bias"], h0=inp["h0"], d_last=d_last,
        workspace=workspace, checkpoints=checkpoints)
    torch.cuda.synchronize()
    return g


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_backward_cut_schedule(dt):
    """More tiles than one wave of resident blocks and a last wave at most
    half full: the last wave's tiles are cut at their middle block into work
    items that hand the state and the adjoint over through the workspace.
    du, ddelta, dz and dh0 are bit-identical to the run with every tile
    whole (a workspace of the checkpoints only), from the backward's own
    forward sweep and from the forward scan's checkpoints; the atomic sums
    agree to fp32 rounding; and a row of the cut tiles matches the oracle."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # 3 resident blocks per SM (4 warps, 168 registers): one wave of slots
    # plus 16 more 32-channel tiles, in one batch row
    dim = 32 * (3 * sms + 16)
    w = workloads.custom(1, dim, 16, 100, in_dtype=dt, has_z=True, a_noise=0.1)
    inp = workloads.make_inputs(w, seed=5900, device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5901)
    inp["h0"] = torch.randn(1, dim, 16, generator=gen, device="cuda")
    dy = torch.randn(1, dim, 100, generator=gen, device="cuda")
    d_last = torch.randn(1, dim, 16, generator=gen, device="cuda")
    # the own sweep's two arrays of states, without the cut schedule's area
    ck_bytes = sss.scan_checkpoints(1, dim, 16, 100, "cpu").numel() * 4
    whole_ws = torch.empty(ck_bytes, dtype=torch.uint8, device="cuda")
    g_whole = _bwd_ws(inp, dy, d_last, whole_ws)
    g_cut = _bwd_ws(inp, dy, d_last, None)   # allocates checkpoints + cut area
    exact = ("du", "ddelta", "dz", "dh0")
    for k in exact:
        assert torch.equal(g_cut[k], g_whole[k]), k
    for k in ("dA", "dB", "dC", "dD", "ddelta_bias"):
        assert norm_err(g_cut[k].cpu().numpy(), g_whole[k].double().cpu().numpy()) <= 1e-5, k
    # from the forward scan's checkpoints: cut (workspace) against whole (none)
    ck = sss.scan_checkpoints(1, dim, 16, 100, "cuda")
    sss.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                           z=inp["z"], delta_bias=inp["delta_bias"], h0=inp["h0"],
                           checkpoints=ck)
    g_ck_whole = _bwd_ws(inp, dy, d_last, False, checkpoints=ck)
    g_ck_cut = _bwd_ws(inp, dy, d_last, None, checkpoints=ck)
    for k in exact:
        assert torch.equal(g_ck_cut[k], g_ck_whole[k]), k
        assert torch.equal(g_ck_cut[k], g_whole[k]), k
    # the cut tiles (the last 16) against the oracle: their channels only
    c0 = dim - 32 * 16
    sub = {k: (v[:, c0:] if v is not None and v.dim() == 3 else v) for k, v in inp.items()}
    sub["A"] = inp["A"][c0:]
    for k in ("D", "delta_bias"):
        sub[k] = inp[k][c0:] if inp[k] is not None else None
    sub["B"], sub["C"] = inp["B"], inp["C"]
    h = workloads.to_numpy_f64(sub)
    g_ref = oracle.selective_scan_bwd(
        h["u"], h["delta"], h["A"], h["B"], h["C"], dy[:, c0:].double().cpu().numpy(),
        D=h["D"], z=h["z"], delta_bias=h["delta_bias"], delta_softplus=True, h0=h["h0"],
        d_last=d_last[:, c0:].double().cpu().numpy())
    for k in ("du", "ddelta", "dz", "dh0"):
        assert norm_err(g_cut[k][:, c0:].cpu().numpy(), g_ref[k]) <= TOL, k
    for k in ("dA", "dD", "ddelta_bias"):
        assert norm_err(g_cut[k][c0:].cpu().numpy(), g_ref[k]) <= TOL, k


def test_backward_cut_schedule_with_eight_states():
    """The cut schedule with 8 states (two warps per block, so more blocks
    per SM): the smallest whole number of 32-channel tiles for which the
    workspace size asks for the cut area, then the cut run against the whole
    run (bit-identical du, ddelta, dz, dh0)."""
    lib = sss.load_library()
    ck_bytes = lambda dim: sss.scan_checkpoints(1, dim, 8, 48, "cpu").numel() * 4

    def need(dim):
        a = sss.ScanBwdArgs()
        a.batch, a.dim, a.dstate, a.seqlen = 1, dim, 8, 48
        a.in_dtype = sss.MSS_BF16
        for f in ("u", "delta", "A", "B", "C", "dy", "du", "ddelta", "dA", "dB", "dC"):
            setattr(a, f, 256)
        n = ctypes.c_size_t(0)
        assert lib.mss_scan_bwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == sss.MSS_OK
        return n.value

    sms = torch.cuda.get_device_properties(0).multi_processor_count
    dim = next(32 * k for k in range(sms, 32 * sms) if need(32 * k) > ck_bytes(32 * k))
    w = workloads.custom(1, dim, 8, 48, in_dtype="bf16", has_z=True, a_noise=0.1)
    inp = workloads.make_inputs(w, seed=5910, device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5911)
    inp["h0"] = torch.randn(1, dim, 8, generator=gen, device="cuda")
    dy = torch.randn(1, dim, 48, generator=gen, device="cuda")
    d_last = torch.randn(1, dim, 8, generator=gen, device="cuda")
    whole_ws = torch.empty(ck_bytes(dim), dtype=torch.uint8, device="cuda")
    g_whole = _bwd_ws(inp, dy, d_last, whole_ws)
    g_cut = _bwd_ws(inp, dy, d_last, None)
    for k in ("du", "ddelta", "dz", "dh0"):
        assert torch.equal(g_cut[k], g_whole[k]), k
    for k in ("dA", "dB", "dC", "dD", "ddelta_bias"):
        assert norm_err(g_cut[k].cpu().numpy(), g_whole[k].double().cpu().numpy()) <= 1e-5, k
