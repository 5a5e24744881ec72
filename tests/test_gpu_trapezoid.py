"""The three-term trapezoidal update on the GPU (needs a GPU).

h_t = a_t h_{t-1} + Delta_t / 2 (a_t B_{t-1} u_{t-1} + B_t u_t): the CUDA
path against the fp64 oracle (whose trapezoidal update is pinned on the CPU
by its no-decay closed form and its second-order convergence).  Cases cover
the previous step crossing 16-step blocks, sequence chunks of split plans
(where a chunk reads the step before it from HBM), ragged lengths, fewer
than 16 states, h0 / last_state, strided views and the plain-load path.
"""
import pytest
import torch

import selective_state_space_48_b200 as sss
import workloads
from scan_checks import gpu_inputs, norm_err, tolerance

pytestmark = pytest.mark.gpu


def _oracle(w, inp):
    import oracle
    h = workloads.to_numpy_f64(inp)
    return oracle.selective_scan(
        h["u"], h["delta"], h["A"], h["B"], h["C"], D=h["D"], z=h["z"],
        delta_bias=h["delta_bias"], delta_softplus=w.softplus, h0=h["h0"],
        return_last_state=True, trapezoid=True)


CASES = [
    # name, batch, dim, N, L, dtype, splits
    ("bf16", 2, 80, 16, 1000, "bf16", 0),
    ("f32-N5-ragged", 2, 40, 5, 333, "f32", 0),
    ("bf16-split3", 1, 64, 16, 3001, "bf16", 3),
    ("f32-split7", 1, 32, 16, 4999, "f32", 7),
    ("f32-plain-loads", 1, 48, 16, 301, "f32", 0),  # 301 * 4 B rows: no TMA
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_trapezoid_matches_the_oracle(case):
    name, batch, dim, N, L, dt, splits = case
    w = workloads.custom(batch, dim, N, L, in_dtype=dt, has_z=True, a_noise=0.1)
    inp = gpu_inputs(w, seed=5300 + len(name), h0=True)
    y, last = sss.selective_scan_fwd(
        inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"], z=inp["z"],
        delta_bias=inp["delta_bias"], h0=inp["h0"], return_last_state=True,
        plan_splits=splits, trapezoid=True, check_status=True)
    torch.cuda.synchronize()
    y_ref, last_ref = _oracle(w, inp)
    tol = tolerance(w.in_dtype)
    assert norm_err(y.cpu().numpy(), y_ref) <= tol, name
    assert norm_err(last.cpu().numpy(), last_ref) <= tol, name


def test_trapezoid_on_strided_views():
    """u and z as the halves of one projection: the step before each block
    is read through the strides."""
    w = workloads.custom(2, 48, 16, 640, in_dtype="bf16", has_z=True)
    inp = gpu_inputs(w, seed=5350, h0=False)
    xz = torch.cat([inp["u"], inp["z"]], dim=1)
    u, z = xz[:, :48], xz[:, 48:]
    y = sss.selective_scan_fwd(u, inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                               z=z, delta_bias=inp["delta_bias"], trapezoid=True,
                               plan_splits=2, check_status=True)
    torch.cuda.synchronize()
    y_ref, _ = _oracle(w, inp)
    assert norm_err(y.cpu().numpy(), y_ref) <= tolerance("bf16")


def test_trapezoid_differs_from_euler():
    """The flag changes the result (the two updates are not the same map)."""
    w = workloads.custom(1, 32, 16, 200, in_dtype="f32", has_z=False)
    inp = gpu_inputs(w, seed=5351, h0=False)
    args = dict(D=inp["D"], delta_bias=inp["delta_bias"])
    y1 = sss.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], **args)
    y2 = sss.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                trapezoid=True, **args)
    torch.cuda.synchronize()
    assert float((y1 - y2).abs().max()) > 1e-3 * float(y1.abs().max())


def test_trapezoid_at_the_130m_layer_shape_every_element():
    """The trapezoidal update at the shape `bench.py --trapezoid` times
    (Mamba-130M layer, bf16 inputs), every output element against the
    oracle."""
    from scan_checks import compare_all_channels, run_gpu
    w = workloads.BY_NAME["mamba130m-layer"]
    inp = gpu_inputs(w)
    y = run_gpu(w, inp, trapezoid=True, check_status=True)
    st = compare_all_channels(w, inp, y, trapezoid=True)
    assert st.norm_err <= tolerance(w.in_dtype), st.summary()
