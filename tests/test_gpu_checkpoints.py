"""Forward-scan checkpoints for the backward pass (needs a GPU).

With mss_scan_args.checkpoints the forward scan also writes the state of
every channel at the start of every 16-step block and, in a second array,
the state entering its 9th step; the backward pass starts from them
instead of its own forward sweep.  Checked: the checkpoints are the
oracle's state after the first 16 k (and 16 k + 8) steps (its last state
of the prefix); y does not change; the backward from checkpoints matches
the backward without them and the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_48_b200 as sss
import workloads
from scan_checks import gpu_inputs, norm_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,dt", [(16, "bf16"), (5, "f32")])
def test_checkpoints_are_the_prefix_states(N, dt):
    batch, dim, L = 2, 40, 200
    w = workloads.custom(batch, dim, N, L, in_dtype=dt, has_z=True)
    inp = gpu_inputs(w, seed=5400 + N, h0=True)
    ck = sss.scan_checkpoints(batch, dim, N, L, "cuda")
    kw = dict(D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"], h0=inp["h0"])
    y1 = sss.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                checkpoints=ck, check_status=True, **kw)
    y0 = sss.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], **kw)
    torch.cuda.synchronize()
    assert torch.equal(y1, y0)
    NP = 4 * {1: 1, 2: 2}.get((N + 3) // 4, 4)
    tiles, nblk = batch * ((dim + 31) // 32), (L + 15) // 16
    c2 = ck.view(2, tiles, nblk, NP, 32).cpu().numpy()
    h = workloads.to_numpy_f64(inp)
    for k, arr in ((0, 0), (1, 0), (5, 0), (nblk - 1, 0), (0, 1), (3, 1), (nblk - 2, 1)):
        c = c2[arr]
        t = 16 * k + 8 * arr
        if t == 0:
            want = h["h0"]
        else:
            _, want = oracle.selective_scan(
                h["u"][..., :t], h["delta"][..., :t], h["A"], h["B"][..., :t],
                h["C"][..., :t], D=h["D"], z=h["z"][..., :t], delta_bias=h["delta_bias"],
                h0=h["h0"], return_last_state=True)
        got = np.zeros_like(want)
        for b in range(batch):
            for d in range(dim):
                tile = b * ((dim + 31) // 32) + d // 32
                got[b, d] = c[tile, k, :N, d % 32]
        assert norm_err(got, want) <= 2e-3, (k, arr)


def test_backward_from_checkpoints():
    batch, dim, N, L = 2, 48, 16, 500
    w = workloads.custom(batch, dim, N, L, in_dtype="bf16", has_z=True, a_noise=0.1)
    inp = gpu_inputs(w, seed=5450, h0=True)
    dy = torch.randn(batch, dim, L, device="cuda")
    kw = dict(D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"], h0=inp["h0"])
    ck = sss.scan_checkpoints(batch, dim, N, L, "cuda")
    sss.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                           checkpoints=ck, **kw)
    g1 = sss.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy,
                                checkpoints=ck, **kw)
    g0 = sss.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy, **kw)
    torch.cuda.synchronize()
    h = workloads.to_numpy_f64(inp)
    g_ref = oracle.selective_scan_bwd(h["u"], h["delta"], h["A"], h["B"], h["C"],
                                      dy.double().cpu().numpy(), D=h["D"], z=h["z"],
                                      delta_bias=h["delta_bias"], h0=h["h0"])
    for k in ("du", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias", "dh0"):
        a, b = g1[k].cpu().numpy(), g0[k].cpu().numpy()
        assert norm_err(a, b) <= 1e-6, k
        assert norm_err(a, g_ref[k]) <= 1e-4, k
