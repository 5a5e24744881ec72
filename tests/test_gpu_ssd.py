"""Mamba-2 (SSD) chunked scan on the tensor cores against the fp64 oracle
(needs a GPU).

The oracle is the sequential recurrence with a scalar A per head (pinned on
the CPU by the quadratic masked form and by its reduction to the S6 scan).
The CUDA path evaluates the same map by 128-step chunks of bf16 matrix
products with fp32 accumulation, so its tolerance comes from bf16
rounding, not fp32: the decayed scores S', the weighted inputs X'' and
the carried state h_prev each enter one product rounded to bf16 (unit
roundoff u = 2^-8, relative error at most u per operand).  An output is a
sum of such products whose rounding errors are independent and of either
sign, so its error is a random sum of per-term errors, each within u of
its term; for a sum of terms of random sign the error stays below
u * max |y| except far in the tails.  The bound used is u (rounded up to
4e-3) of max |y| (and of max |h| for the final state), with another 2^-8
when y itself is stored in bf16.  tests/test_ssd_chunked_model.py runs the
same decomposition with the same three roundings in fp64 on the CPU and
stays at 1.5e-3 to 3.5e-3 on its cases.

Cases: chunks with a ragged tail, a single short chunk, two groups of B
and C, no optional inputs with softplus off, an initial state, bf16 output,
a long carry chain, and every element of the full 2.7B-layer shape.
"""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_48_b200 as sss
import workloads
from oracle.compare import ErrorStats
from scan_checks import norm_err

pytestmark = pytest.mark.gpu

U_BF16 = 2.0 ** -8
TOL = 4e-3  # u = 2^-8 = 3.9e-3, rounded up


def _oracle(inp, softplus=True, heads=None, batch=None):
    h = workloads.to_numpy_f64(inp)
    x, dt, A, z, h0 = h["x"], h["dt"], h["A"], h["z"], h["h0"]
    B, C, D, bias = h["B"], h["C"], h["D"], h["dt_bias"]
    if batch is not None:
        sel = slice(batch, batch + 1)
        x, dt, B, C = x[sel], dt[sel], B[sel], C[sel]
        z = None if z is None else z[sel]
        h0 = None if h0 is None else h0[sel]
    if heads is not None:  # a subset of heads of a one-group input
        assert B.shape[2] == 1
        x, dt, A = x[:, :, heads], dt[:, :, heads], A[heads]
        z = None if z is None else z[:, :, heads]
        D = None if D is None else D[heads]
        bias = None if bias is None else bias[heads]
        h0 = None if h0 is None else h0[:, heads]
    return oracle.ssd_scan(x, dt, A, B, C, D=D, z=z, dt_bias=bias, dt_softplus=softplus,
                           h0=h0, return_last_state=True)


def _run(inp, softplus=True, out_dtype=torch.float32):
    return sss.ssd_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                       z=inp["z"], dt_bias=inp["dt_bias"], dt_softplus=softplus,
                       h0=inp["h0"], return_last_state=True, out_dtype=out_dtype,
                       check_status=True)


CASES = [
    # name, batch, L, heads, groups, z, h0
    ("ragged-3-chunks-2-groups", 2, 300, 4, 2, True, True),
    ("one-short-chunk", 1, 50, 2, 1, True, False),
    ("two-full-chunks", 1, 256, 3, 1, False, True),
    ("long-carry", 1, 2000, 2, 1, True, False),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_ssd_matches_the_oracle(case):
    name, batch, L, H, G, has_z, h0 = case
    w = workloads.SsdWorkload(name, batch, L, H, ngroups=G, has_z=has_z)
    inp = workloads.make_ssd_inputs(w, seed=5700 + L, device="cuda", h0=h0)
    y, last = _run(inp)
    torch.cuda.synchronize()
    y_ref, last_ref = _oracle(inp)
    assert norm_err(y.cpu().numpy(), y_ref) <= TOL, name
    assert norm_err(last.cpu().numpy(), last_ref) <= TOL, name


def test_ssd_without_optional_inputs_and_softplus_off():
    w = workloads.SsdWorkload("plain", 1, 200, 2, has_z=False, has_D=False,
                              has_dt_bias=False, softplus=False)
    inp = workloads.make_ssd_inputs(w, seed=5750, device="cuda")
    # positive steps without softplus
    inp["dt"] = (inp["dt"].float().abs() * 0.05 + 0.001).to(torch.bfloat16)
    y, last = _run(inp, softplus=False)
    torch.cuda.synchronize()
    y_ref, last_ref = _oracle(inp, softplus=False)
    assert norm_err(y.cpu().numpy(), y_ref) <= TOL
    assert norm_err(last.cpu().numpy(), last_ref) <= TOL


def test_ssd_bf16_output():
    w = workloads.SsdWorkload("bf16-out", 1, 300, 2, has_z=True)
    inp = workloads.make_ssd_inputs(w, seed=5751, device="cuda", h0=True)
    y, _ = _run(inp, out_dtype=torch.bfloat16)
    yf, _ = _run(inp)
    torch.cuda.synchronize()
    assert y.dtype == torch.bfloat16
    assert torch.equal(y, yf.to(torch.bfloat16))
    y_ref, _ = _oracle(inp)
    assert norm_err(y.float().cpu().numpy(), y_ref) <= TOL + U_BF16


def test_ssd_full_layer_every_element():
    """The 2.7B-layer shape in the launch configuration the bench times,
    with an initial state: every element of y and of the final state
    against the oracle (run one batch row at a time)."""
    w = workloads.SSD_BY_NAME["mamba2-2.7b-layer"]
    inp = workloads.make_ssd_inputs(w, seed=5752, device="cuda", h0=True)
    y, last = _run(inp)
    torch.cuda.synchronize()
    assert torch.isfinite(y).all()
    sy, sl = ErrorStats(), ErrorStats()
    for b in range(w.batch):
        y_ref, last_ref = _oracle(inp, batch=b)
        sy.add(y[b:b + 1].cpu().numpy(), y_ref)
        sl.add(last[b:b + 1].cpu().numpy(), last_ref)
    assert sy.count == y.numel() and sl.count == last.numel()
    assert sy.norm_err <= TOL, sy.summary()
    assert sl.norm_err <= TOL, sl.summary()


def test_ssd_is_deterministic():
    w = workloads.SsdWorkload("det", 2, 700, 3, has_z=True)
    inp = workloads.make_ssd_inputs(w, seed=5753, device="cuda", h0=True)
    y1, l1 = _run(inp)
    y2, l2 = _run(inp)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(l1, l2)


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


CUT_CASES = [
    # name, batch, L, heads, groups: with 148 SMs, the sequences of the last
    # wave are cut into pieces spread over the schedule
    ("three-pieces-ragged", 2, 657, 160, 2),   # 320: 2 waves + 24, 3 pieces of 2 chunks
    ("halves-of-two-chunks", 1, 129, 160, 1),  # 160: 1 wave + 12, 2 pieces of 1 chunk
    ("halves-of-five-chunks", 1, 640, 200, 1), # 200: 1 wave + 52, pieces of 2 and 3 chunks
    ("four-pieces-of-one-chunk", 4, 385, 112, 1),  # 448: 3 waves + 4, 4 pieces
]


@pytest.mark.parametrize("case", CUT_CASES, ids=[c[0] for c in CUT_CASES])
def test_ssd_cut_sequences_equal_the_whole_schedule(case):
    """Sequences cut into pieces at chunk boundaries (each piece starting
    from the fp32 end state of the piece before) run the same per-chunk
    arithmetic as the whole sequence, so y and the final state are
    bit-identical to the schedule without a workspace; and they match the
    oracle."""
    name, batch, L, H, G = case
    w = workloads.SsdWorkload(name, batch, L, H, ngroups=G, has_z=True)
    inp = workloads.make_ssd_inputs(w, seed=5760 + L, device="cuda", h0=True)
    args = sss.make_ssd_args(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"])
    assert sss.ssd_workspace_size(args) > 0 or _sms() != 148
    y_cut, last_cut = _run(inp)
    y_whole, last_whole = sss.ssd_fwd(
        inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], D=inp["D"], z=inp["z"],
        dt_bias=inp["dt_bias"], h0=inp["h0"], return_last_state=True, check_status=True,
        workspace=False)
    torch.cuda.synchronize()
    assert torch.equal(y_cut, y_whole)
    assert torch.equal(last_cut, last_whole)
    y_ref, last_ref = _oracle(inp)
    assert norm_err(y_cut.cpu().numpy(), y_ref) <= TOL
    assert norm_err(last_cut.cpu().numpy(), last_ref) <= TOL


def test_ssd_workspace_plan():
    """What is cut, and the workspace it takes: nothing without a whole wave
    to run between the pieces, for one chunk, or when the last wave is more
    than half full; r sequences in min(round(SMs / r), waves + 1, chunks, 8)
    pieces otherwise.  A workspace smaller than asked for is rejected before
    launch."""
    sms = _sms()

    def need(batch, H, L):
        w = workloads.SsdWorkload("plan", batch, L, H, has_z=False)
        inp = workloads.make_ssd_inputs(w, seed=5770, device="cuda")
        args = sss.make_ssd_args(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"])
        return sss.ssd_workspace_size(args), inp

    state = 64 * 128 * 4
    assert need(1, 4, 300)[0] == 0               # less than one wave
    assert need(1, sms + 6, 128)[0] == 0         # one chunk
    assert need(1, sms, 300)[0] == 0             # whole waves
    assert need(1, 2 * sms - 1, 300)[0] == 0     # last wave more than half full
    assert need(1, 2 * sms + 24, 640)[0] == 512 + 2 * 24 * state  # 3 pieces
    n, inp = need(1, sms + 6, 300)
    assert n == 512 + 6 * state                  # 2 pieces: counter, flags, 6 states
    small = torch.empty(n - 4, dtype=torch.uint8, device="cuda")
    with pytest.raises(sss.MssError) as ex:
        sss.ssd_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], workspace=small)
    assert ex.value.code == sss.MSS_ERR_WORKSPACE
