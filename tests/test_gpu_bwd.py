"""Backward scan against the fp64 oracle backward (needs a GPU).

The oracle's gradients are pinned by central finite differences of the
forward oracle on the CPU.  Here every gradient of the CUDA backward (du,
ddelta, dA, dB, dC, dD, dz, ddelta_bias, dh0) is compared with the oracle on
the same inputs (bf16 cases: the oracle reads the same bf16-rounded values),
as max |g_gpu - g_ref| / max |g_ref| per tensor.  Both sides do the same
arithmetic; the GPU does it in fp32 with atomic sums over channels and
batch rows, hence the fp32-level bound.
"""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_48_b200 as sss
import workloads
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
