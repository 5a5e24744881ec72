"""Parity of the CUDA selective scan with the fp64 oracle (needs a GPU).

Every test calls the library through its C ABI (ctypes binding) and
compares with the oracle on the same seeded inputs at the tolerances stated
in scan_checks.py.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import pins
import selective_state_space_48_b200 as sss
import workloads
from scan_checks import (compare_all_channels, gpu_inputs, norm_err, run_gpu,
                         run_oracle, tolerance)

pytestmark = pytest.mark.gpu


def test_tiny_fp32_workload_matches_oracle():
    w = workloads.BY_NAME["tiny-fp32"]
    inp = gpu_inputs(w)
    y, last = run_gpu(w, inp, return_last_state=True)
    want, want_last = run_oracle(w, inp, return_last_state=True)
    assert norm_err(y.cpu(), want) <= tolerance(w.in_dtype)
    assert norm_err(last.cpu(), want_last) <= tolerance(w.in_dtype)


ODD = [
    # batch, dim, N, L, dtype, z, D, bias, softplus, h0
    (1, 1, 1, 1, "f32", False, False, False, True, False),
    (1, 3, 4, 7, "f32", True, True, True, True, True),
    (2, 3, 5, 33, "bf16", True, True, True, True, False),
    (1, 33, 16, 255, "f32", True, True, True, True, True),
    (2, 33, 16, 257, "bf16", True, False, True, True, True),
    (1, 64, 8, 100, "f32", False, True, False, False, False),
    (2, 40, 13, 129, "f32", True, True, True, True, True),
    (1, 5, 2, 4097, "bf16", True, True, True, True, False),
    (3, 1, 16, 31, "f32", True, True, True, True, True),
]


@pytest.mark.parametrize("case", ODD, ids=lambda c: "b{}d{}n{}l{}{}".format(*c[:5]))
def test_odd_shapes_match_oracle(case):
    batch, dim, N, L, dt, z, D, bias, sp, h0 = case
    w = workloads.custom(batch, dim, N, L, in_dtype=dt, has_z=z, has_D=D,
                         has_delta_bias=bias, softplus=sp)
    inp = gpu_inputs(w, seed=sum(case[:4]), h0=h0)
    if not sp:
        # without softplus the step must stay positive: use |delta|
        inp["delta"] = inp["delta"].abs() * 0.5
    y, last = run_gpu(w, inp, return_last_state=True)
    want, want_last = run_oracle(w, inp, return_last_state=True)
    tol = tolerance(dt)
    assert norm_err(y.cpu(), want) <= tol
    assert norm_err(last.cpu(), want_last) <= tol


@pytest.mark.parametrize("splits", [2, 3, 7, 64])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("N,L", [(16, 5000), (5, 4999), (2, 3001)])
def test_sequence_split_matches_oracle(splits, dt, N, L):
    """Chunks combined through their carries give the sequential result ("The relay":
    group the steps any way you like).  Odd lengths take the plain-load
    path, N < 16 the kernels with fewer state groups."""
    w = workloads.custom(2, 40, N, L, in_dtype=dt, has_z=True)
    inp = gpu_inputs(w, seed=splits + N, h0=True)
    y, last = run_gpu(w, inp, plan_splits=splits, return_last_state=True,
                      check_status=True)
    want, want_last = run_oracle(w, inp, return_last_state=True)
    tol = tolerance(dt)
    assert norm_err(y.cpu(), want) <= tol
    assert norm_err(last.cpu(), want_last) <= tol


def test_split_with_slow_decay_matches_oracle():
    """Tiny steps (Delta ~ 1e-3) keep the carried state alive through whole
    chunks, so the carry correction must run to the end of the chunk."""
    w = workloads.custom(1, 32, 16, 6000, in_dtype="f32", has_z=True)
    inp = gpu_inputs(w, seed=5, h0=True)
    inp["delta_bias"] = torch.full_like(inp["delta_bias"], -7.0)
    y = run_gpu(w, inp, plan_splits=6, check_status=True)
    want = run_oracle(w, inp)
    assert norm_err(y.cpu(), want) <= tolerance("f32")


@pytest.mark.parametrize("dt,out", [("f32", torch.float32), ("bf16", torch.bfloat16)])
def test_carry_across_many_segments(dt, out):
    """Slow decay (Delta ~ 1e-3) over chunks of 2 600 steps: the carried
    state stays alive across several 512-step segments of the carry launch,
    the last of them ragged; the final state comes from the chunk prefix."""
    w = workloads.custom(2, 40, 16, 7777, in_dtype=dt, has_z=True, a_noise=0.1)
    inp = gpu_inputs(w, seed=9, h0=True)
    inp["delta_bias"] = torch.full_like(inp["delta_bias"], -7.0)
    y, last = run_gpu(w, inp, out_dtype=out, plan_splits=3, return_last_state=True,
                      check_status=True)
    want, want_last = run_oracle(w, inp, return_last_state=True)
    assert norm_err(y.float().cpu(), want) <= tolerance(dt, out)
    assert norm_err(last.cpu(), want_last) <= tolerance(dt)


@pytest.mark.parametrize("name", ["mamba130m-layer", "mamba1.4b-layer",
                                  "long-context", "audio-length"])
def test_full_size_workload_every_element(name):
    """The bench's launch configuration (automatic plan) at full size:
    every output element against the fp64 oracle (run on all channels, a
    block at a time), and a run grouped into a different number of
    sequence chunks, also against the oracle (any grouping gives the same
    result, "The relay")."""
    w = workloads.BY_NAME[name]
    inp = gpu_inputs(w)
    y = run_gpu(w, inp, check_status=True)
    tol = tolerance(w.in_dtype)
    st = compare_all_channels(w, inp, y)
    assert st.count == w.batch * w.dim * w.seqlen
    assert st.norm_err <= tol, st.summary()
    other = 5 if w.seqlen >= 5 * 1024 else 2
    y2 = run_gpu(w, inp, plan_splits=other, check_status=True)
    st2 = compare_all_channels(w, inp, y2)
    assert st2.norm_err <= tol, st2.summary()
    del y, y2, inp
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["mamba130m-layer", "mamba1.4b-layer"])
def test_full_size_bf16_output_every_element(name):
    """bf16 y on the layer workloads, every element against the oracle."""
    w = workloads.BY_NAME[name]
    inp = gpu_inputs(w)
    y = run_gpu(w, inp, out_dtype=torch.bfloat16, check_status=True)
    st = compare_all_channels(w, inp, y)
    assert st.norm_err <= tolerance(w.in_dtype, torch.bfloat16), st.summary()
    del y, inp
    torch.cuda.empty_cache()


def test_resume_from_last_state():
    w = workloads.custom(2, 48, 16, 700, in_dtype="f32", has_z=True)
    inp = gpu_inputs(w, seed=21, h0=True)
    y, last = run_gpu(w, inp, return_last_state=True)
    cut = 333
    p1 = dict(inp)
    p2 = dict(inp)
    for k in ("u", "delta", "z", "B", "C"):
        p1[k] = inp[k][..., :cut].contiguous()
        p2[k] = inp[k][..., cut:].contiguous()
    w1 = workloads.custom(2, 48, 16, cut, in_dtype="f32", has_z=True)
    w2 = workloads.custom(2, 48, 16, 700 - cut, in_dtype="f32", has_z=True)
    y1, s1 = run_gpu(w1, p1, return_last_state=True)
    p2["h0"] = s1
    y2, s2 = run_gpu(w2, p2, return_last_state=True)
    assert torch.allclose(torch.cat([y1, y2], -1), y, rtol=1e-5, atol=1e-5)
    assert torch.allclose(s2, last, rtol=1e-5, atol=1e-5)


def test_single_step_scan_equals_state_update():
    w = workloads.custom(3, 50, 16, 1, in_dtype="f32", has_z=True)
    inp = gpu_inputs(w, seed=8, h0=True)
    y, last = run_gpu(w, inp, return_last_state=True)
    st = inp["h0"].clone()
    yu = sss.selective_state_update(st, inp["u"][..., 0].contiguous(),
                                    inp["delta"][..., 0].contiguous(), inp["A"],
                                    inp["B"][..., 0].contiguous(),
                                    inp["C"][..., 0].contiguous(), D=inp["D"],
                                    z=inp["z"][..., 0].contiguous(),
                                    dt_bias=inp["delta_bias"])
    assert torch.allclose(yu, y[..., 0], rtol=1e-5, atol=1e-6)
    assert torch.allclose(st, last, rtol=1e-5, atol=1e-6)


def test_relay_worked_example_through_the_abi():
    """(0.6, 0.4) then (0.5, 1.0) = (0.3, 1.2), realised with N = 1, D = 0,
    C = 1, softplus off: y = (0.6 x + 0.4, 0.3 x + 1.2)."""
    g = pins.load_golden("relay_worked_example.txt")
    x0 = 2.5
    u, delta, A, B, C, h0 = pins._worked_example_inputs(g, x0)
    dev = lambda a: torch.tensor(a, dtype=torch.float32, device="cuda").contiguous()
    y, last = sss.selective_scan_fwd(dev(u), dev(delta), dev(A), dev(B), dev(C),
                                     delta_softplus=False, h0=dev(h0),
                                     return_last_state=True)
    want = [g["after_step1_fade"] * x0 + g["after_step1_add"], g["a12"] * x0 + g["b12"]]
    assert np.allclose(y[0, 0].cpu().numpy(), want, rtol=2e-6)
    assert abs(last.item() - want[1]) <= 2e-6 * abs(want[1])


def test_bf16_output():
    w = workloads.custom(2, 64, 16, 777, in_dtype="bf16", has_z=True)
    inp = gpu_inputs(w, seed=3)
    y = run_gpu(w, inp, out_dtype=torch.bfloat16)
    assert y.dtype == torch.bfloat16
    want = run_oracle(w, inp)
    assert norm_err(y.float().cpu(), want) <= tolerance("bf16", torch.bfloat16)
    y2 = run_gpu(w, inp, out_dtype=torch.bfloat16, plan_splits=3)
    assert norm_err(y2.float().cpu(), want) <= tolerance("bf16", torch.bfloat16)


def test_unsplit_scan_is_deterministic():
    w = workloads.custom(2, 96, 16, 1000, in_dtype="bf16", has_z=True)
    inp = gpu_inputs(w, seed=4)
    y1 = run_gpu(w, inp, plan_splits=1)
    y2 = run_gpu(w, inp, plan_splits=1)
    assert torch.equal(y1, y2)


def test_dropped_publish_times_out_and_device_stays_usable():
    """A publication that never comes (test flag): the bounded wait before
    the chunks' carries are composed runs out, the status word says so, and
    the next call works."""
    w = workloads.custom(1, 32, 16, 4096, in_dtype="f32", has_z=False)
    inp = gpu_inputs(w, seed=2)
    with pytest.raises(sss.MssError) as ei:
        run_gpu(w, inp, plan_splits=4, test_flags=sss.MSS_TESTFLAG_DROP_PUBLISH,
                spin_timeout_ns=20_000_000, check_status=True)
    assert ei.value.code == sss.MSS_ERR_TIMEOUT
    y = run_gpu(w, inp, plan_splits=4, check_status=True)
    assert norm_err(y.cpu(), run_oracle(w, inp)) <= tolerance("f32")


def test_invalid_calls_return_codes_on_device():
    w = workloads.custom(1, 8, 16, 64, in_dtype="f32")
    inp = gpu_inputs(w)
    args = sss.make_scan_args(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                              y=torch.empty(1, 8, 64, device="cuda"))
    args.dstate = 20
    lib = sss.load_library()
    import ctypes
    assert lib.mamba_selective_scan_fwd(ctypes.byref(args), None) == sss.MSS_ERR_UNSUPPORTED
    torch.cuda.synchronize()


@pytest.mark.parametrize("dt,N", [("f32", 16), ("bf16", 16), ("f32", 5)])
def test_state_update_matches_oracle(dt, N):
    batch, dim = 3, 70
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    g = torch.Generator(device="cuda")
    g.manual_seed(77 + N)
    r = lambda *s: torch.randn(*s, generator=g, device="cuda")
    state = r(batch, dim, N)
    x, dtv, z = r(batch, dim).to(tdt), r(batch, dim).to(tdt), r(batch, dim).to(tdt)
    A = -torch.rand(dim, N, generator=g, device="cuda") * 3
    B, C = r(batch, N).to(tdt), r(batch, N).to(tdt)
    D, bias = r(dim), r(dim) * 0.5
    st_ref, y_ref = oracle.selective_state_update(
        state.cpu().double().numpy(), x.cpu().double().numpy(), dtv.cpu().double().numpy(),
        A.cpu().double().numpy(), B.cpu().double().numpy(), C.cpu().double().numpy(),
        D=D.cpu().double().numpy(), z=z.cpu().double().numpy(),
        dt_bias=bias.cpu().double().numpy())
    st = state.clone()
    y = sss.selective_state_update(st, x, dtv, A, B, C, D=D, z=z, dt_bias=bias)
    tol = 1e-5
    assert norm_err(y.cpu(), y_ref) <= tol
    assert norm_err(st.cpu(), st_ref) <= tol


def test_state_update_past_the_grid_row_limit():
    """More than 65535 batch rows: the 16-state kernel runs on a flat grid
    of channels instead of one grid row per batch row; the result still
    matches the oracle."""
    batch, dim, N = 65537, 3, 16
    g = torch.Generator(device="cuda")
    g.manual_seed(93)
    r = lambda *s: torch.randn(*s, generator=g, device="cuda")
    state = r(batch, dim, N)
    x, dtv, z = r(batch, dim), r(batch, dim), r(batch, dim)
    A = -torch.rand(dim, N, generator=g, device="cuda") * 3
    B, C = r(batch, N), r(batch, N)
    D, bias = r(dim), r(dim) * 0.5
    st_ref, y_ref = oracle.selective_state_update(
        state.cpu().double().numpy(), x.cpu().double().numpy(), dtv.cpu().double().numpy(),
        A.cpu().double().numpy(), B.cpu().double().numpy(), C.cpu().double().numpy(),
        D=D.cpu().double().numpy(), z=z.cpu().double().numpy(),
        dt_bias=bias.cpu().double().numpy())
    st = state.clone()
    y = sss.selective_state_update(st, x, dtv, A, B, C, D=D, z=z, dt_bias=bias)
    assert norm_err(y.cpu(), y_ref) <= 1e-5
    assert norm_err(st.cpu(), st_ref) <= 1e-5


def test_state_update_with_unaligned_B_C_takes_the_general_path():
    """B and C starting off a 16-byte boundary use the scalar path; the
    result is the same as from aligned copies."""
    batch, dim, N = 2, 64, 16
    g = torch.Generator(device="cuda")
    g.manual_seed(91)
    r = lambda *s: torch.randn(*s, generator=g, device="cuda")
    state = r(batch, dim, N)
    x, dtv = r(batch, dim), r(batch, dim)
    A = -torch.rand(dim, N, generator=g, device="cuda") * 3
    flatB, flatC = r(batch * N + 1), r(batch * N + 1)
    B_off, C_off = flatB[1:].view(batch, N), flatC[1:].view(batch, N)
    assert B_off.data_ptr() % 16 != 0
    s1, s2 = state.clone(), state.clone()
    y1 = sss.selective_state_update(s1, x, dtv, A, B_off, C_off)
    y2 = sss.selective_state_update(s2, x, dtv, A, B_off.clone(), C_off.clone())
    torch.cuda.synchronize()
    assert torch.allclose(y1, y2, rtol=1e-6, atol=1e-6)
    assert torch.allclose(s1, s2, rtol=1e-6, atol=1e-6)
