"""Packed independent sequences (cu_seqlens) on the GPU (needs a GPU).

Every batch row holds several sequences; the state restarts from zero at
each interior offset.  The CUDA path is compared with the fp64 oracle on the
same offsets (the oracle's restarts are pinned to per-sequence closed forms
on the CPU), with offsets that fall inside 16-step blocks, on block edges,
on sequence-chunk edges of split plans, with 1-step and empty sequences,
and with A entries equal to zero.  A packed row also has to match separate
scans of its sequences.
"""
import numpy as np
import pytest
import torch

import selective_state_space_48_b200 as sss
import workloads
from scan_checks import gpu_inputs, norm_err, run_oracle, tolerance

pytestmark = pytest.mark.gpu


def _offsets(L, cuts):
    cu = sorted(set([0, L] + [c for c in cuts if 0 <= c <= L]))
    return cu


def _run(w, inp, cu, plan_splits=0, h0=True):
    cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
    y, last = sss.selective_scan_fwd(
        inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"], z=inp["z"],
        delta_bias=inp["delta_bias"], delta_softplus=w.softplus,
        h0=inp["h0"] if h0 else None, return_last_state=True,
        plan_splits=plan_splits, cu_seqlens=cu_t, check_status=True)
    torch.cuda.synchronize()
    return y, last


def _oracle(w, inp, cu, h0=True):
    h = workloads.to_numpy_f64(inp)
    import oracle
    return oracle.selective_scan(
        h["u"], h["delta"], h["A"], h["B"], h["C"], D=h["D"], z=h["z"],
        delta_bias=h["delta_bias"], delta_softplus=w.softplus,
        h0=h["h0"] if h0 else None, return_last_state=True, cu_seqlens=cu)


CASES = [
    # name, batch, dim, N, L, dtype, cuts, splits
    ("bf16-mixed", 2, 80, 16, 3000, "bf16", [1, 2, 16, 17, 700, 1008, 1009, 2016, 2999], 0),
    ("f32-N5", 2, 40, 5, 1500, "f32", [3, 64, 65, 800, 1499], 0),
    ("bf16-split3", 1, 64, 16, 3000, "bf16", [1, 500, 1008, 1500, 2016, 2017, 2990], 3),
    ("bf16-split7", 1, 48, 16, 5000, "bf16", [7, 720, 721, 1440, 3000, 4999], 7),
    ("f32-many-short", 1, 32, 16, 512, "f32", list(range(0, 512, 5)), 0),
    # two chunks of 4512 steps; restarts on and next to a 512-step segment
    # boundary of the carry launch
    ("bf16-split2-segments", 1, 48, 16, 9000, "bf16", [5024, 5025, 7000], 2),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_packed_sequences_match_the_oracle(case):
    name, batch, dim, N, L, dt, cuts, splits = case
    w = workloads.custom(batch, dim, N, L, in_dtype=dt, has_z=True, a_noise=0.1)
    inp = gpu_inputs(w, seed=4900 + len(name), h0=True)
    cu = _offsets(L, cuts)
    y, last = _run(w, inp, cu, plan_splits=splits)
    y_ref, last_ref = _oracle(w, inp, cu)
    tol = tolerance(w.in_dtype)
    assert norm_err(y.cpu().numpy(), y_ref) <= tol, name
    assert norm_err(last.cpu().numpy(), last_ref) <= tol, name


def test_empty_sequences_and_restart_at_zero():
    """Empty sequences (repeated offsets) restart once; an empty first
    sequence discards h0 (its end state is h0, the next one starts empty)."""
    w = workloads.custom(2, 32, 16, 600, in_dtype="f32", has_z=True)
    inp = gpu_inputs(w, seed=4951, h0=True)
    for cu in ([0, 0, 100, 100, 100, 600], [0, 250, 250, 600]):
        y, last = _run(w, inp, cu)
        y_ref, last_ref = _oracle(w, inp, cu)
        assert norm_err(y.cpu().numpy(), y_ref) <= tolerance("f32"), cu
        assert norm_err(last.cpu().numpy(), last_ref) <= tolerance("f32"), cu


def test_zero_decay_states_restart():
    """A = 0 keeps a state constant between restarts and zeroes it at them."""
    w = workloads.custom(1, 32, 16, 400, in_dtype="f32", has_z=False)
    inp = gpu_inputs(w, seed=4952, h0=True)
    inp["A"][:, ::3] = 0.0
    cu = [0, 37, 160, 161, 400]
    y, last = _run(w, inp, cu)
    y_ref, last_ref = _oracle(w, inp, cu)
    assert np.isfinite(y.cpu().numpy()).all()
    assert norm_err(y.cpu().numpy(), y_ref) <= tolerance("f32")
    assert norm_err(last.cpu().numpy(), last_ref) <= tolerance("f32")


def test_one_sequence_is_the_plain_scan():
    w = workloads.custom(2, 64, 16, 1000, in_dtype="bf16", has_z=True)
    inp = gpu_inputs(w, seed=4953, h0=True)
    y, last = _run(w, inp, [0, 1000])
    y0, last0 = sss.selective_scan_fwd(
        inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"], z=inp["z"],
        delta_bias=inp["delta_bias"], h0=inp["h0"], return_last_state=True)
    torch.cuda.synchronize()
    assert torch.equal(y, y0) and torch.equal(last, last0)


def test_packed_row_equals_separate_scans():
    w = workloads.custom(1, 64, 16, 900, in_dtype="bf16", has_z=True)
    inp = gpu_inputs(w, seed=4954, h0=False)
    cu = [0, 123, 128, 500, 900]
    y, last = _run(w, inp, cu, h0=False)
    for a, b in zip(cu[:-1], cu[1:]):
        part = {k: (v[..., a:b].contiguous() if k in ("u", "delta", "z", "B", "C") else v)
                for k, v in inp.items()}
        yp, lp = sss.selective_scan_fwd(
            part["u"], part["delta"], part["A"], part["B"], part["C"], D=part["D"],
            z=part["z"], delta_bias=part["delta_bias"], return_last_state=True)
        torch.cuda.synchronize()
        scale = float(yp.abs().max())
        assert float((y[..., a:b] - yp).abs().max()) <= 1e-6 * scale, (a, b)
    assert float((last - lp).abs().max()) <= 1e-6 * float(lp.abs().max())


def test_packed_sequences_at_the_130m_layer_shape_every_element():
    """Eight packed sequences per row at the shape `bench.py --varlen 8`
    times (Mamba-130M layer, bf16 inputs; seeded offsets shared by the
    rows), every output element against the oracle."""
    from scan_checks import compare_all_channels, run_gpu
    w = workloads.BY_NAME["mamba130m-layer"]
    inp = gpu_inputs(w)
    rng = np.random.default_rng(48008)
    cuts = rng.choice(np.arange(1, w.seqlen), size=7, replace=False)
    cu = [0] + sorted(int(c) for c in cuts) + [w.seqlen]
    cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
    y = run_gpu(w, inp, cu_seqlens=cu_t, check_status=True)
    st = compare_all_channels(w, inp, y, cu_seqlens=cu)
    assert st.norm_err <= tolerance(w.in_dtype), st.summary()
