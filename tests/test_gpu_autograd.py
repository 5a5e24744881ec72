"""The autograd wrapper selective_scan_fn (needs a GPU): its forward value
and the gradients torch.autograd returns for every input match the fp64
oracle forward and backward on the same inputs."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_48_b200 as sss
import workloads
from scan_checks import gpu_inputs, norm_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_selective_scan_fn_gradients(dt):
    w = workloads.custom(2, 40, 16, 300, in_dtype=dt, has_z=True, a_noise=0.1)
    inp = gpu_inputs(w, seed=5600, h0=True)
    leaves = {k: v.detach().clone().requires_grad_(True)
              for k, v in inp.items() if v is not None}
    y = sss.selective_scan_fn(leaves["u"], leaves["delta"], leaves["A"], leaves["B"],
                              leaves["C"], D=leaves["D"], z=leaves["z"],
                              delta_bias=leaves["delta_bias"], h0=leaves["h0"])
    dy = torch.randn_like(y)
    (y * dy).sum().backward()
    torch.cuda.synchronize()
    h = workloads.to_numpy_f64(inp)
    y_ref = oracle.selective_scan(h["u"], h["delta"], h["A"], h["B"], h["C"], D=h["D"],
                                  z=h["z"], delta_bias=h["delta_bias"], h0=h["h0"])
    tol = 1e-4 if dt == "f32" else 2e-3
    assert norm_err(y.detach().cpu().numpy(), y_ref) <= tol
    g = oracle.selective_scan_bwd(h["u"], h["delta"], h["A"], h["B"], h["C"],
                                  dy.double().cpu().numpy(), D=h["D"], z=h["z"],
                                  delta_bias=h["delta_bias"], h0=h["h0"])
    # bf16 inputs get their gradients rounded to bf16
    gtol = 1e-4 if dt == "f32" else 2.0 ** -8
    for k, gk in (("u", "du"), ("delta", "ddelta"), ("A", "dA"), ("B", "dB"),
                  ("C", "dC"), ("D", "dD"), ("z", "dz"), ("delta_bias", "ddelta_bias"),
                  ("h0", "dh0")):
        got = leaves[k].grad
        assert got is not None and got.dtype == leaves[k].dtype, k
        assert norm_err(got.float().cpu().numpy(), g[gk]) <= gtol, k


def test_selective_scan_fn_packed_sequences_and_views():
    """Packed sequences through the autograd wrapper (the backward runs its
    own forward sweep), with u and z the two halves of one projection: the
    value and every gradient match the oracle with the same packing."""
    batch, dim, N, L = 2, 40, 16, 300
    w = workloads.custom(batch, dim, N, L, in_dtype="f32", has_z=True, a_noise=0.1)
    inp = gpu_inputs(w, seed=5700, h0=True)
    cu = [0, 17, 32, 33, 200, 300]
    cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
    proj = torch.cat([inp["u"], inp["z"]], dim=1).detach().clone().requires_grad_(True)
    leaves = {k: inp[k].detach().clone().requires_grad_(True)
              for k in ("delta", "A", "B", "C", "D", "delta_bias", "h0")}
    u, z = proj[:, :dim], proj[:, dim:]
    y = sss.selective_scan_fn(u, leaves["delta"], leaves["A"], leaves["B"], leaves["C"],
                              D=leaves["D"], z=z, delta_bias=leaves["delta_bias"],
                              h0=leaves["h0"], cu_seqlens=cu_t)
    dy = torch.randn_like(y)
    (y * dy).sum().backward()
    torch.cuda.synchronize()
    h = workloads.to_numpy_f64(inp)
    y_ref = oracle.selective_scan(h["u"], h["delta"], h["A"], h["B"], h["C"], D=h["D"],
                                  z=h["z"], delta_bias=h["delta_bias"], h0=h["h0"],
                                  cu_seqlens=cu)
    assert norm_err(y.detach().cpu().numpy(), y_ref) <= 1e-4
    g = oracle.selective_scan_bwd(h["u"], h["delta"], h["A"], h["B"], h["C"],
                                  dy.double().cpu().numpy(), D=h["D"], z=h["z"],
                                  delta_bias=h["delta_bias"], h0=h["h0"], cu_seqlens=cu)
    gp = proj.grad.cpu().numpy()
    assert norm_err(gp[:, :dim], g["du"]) <= 1e-4
    assert norm_err(gp[:, dim:], g["dz"]) <= 1e-4
    for k, gk in (("delta", "ddelta"), ("A", "dA"), ("B", "dB"), ("C", "dC"), ("D", "dD"),
                  ("delta_bias", "ddelta_bias"), ("h0", "dh0")):
        assert norm_err(leaves[k].grad.cpu().numpy(), g[gk]) <= 1e-4, k
