"""Parity of the scan on strided views (needs a GPU).

The (batch, rows, seqlen) tensors may be views with their own batch and
row strides and a contiguous time dimension.  Each case builds such views
(u and z as the halves of one projection, B and C with padded rows, a B
shared by every batch row, y inside a larger buffer), runs the CUDA path on
them through the C ABI, and compares with the fp64 oracle fed dense copies
of the same values.  Strides that are multiples of 16 bytes take the TMA
load path, the others the plain-load path; both are covered, as are a
split sequence and a bf16 y.
"""
import numpy as np
import pytest
import torch

import selective_state_space_48_b200 as sss
import workloads
from scan_checks import norm_err, run_oracle, tolerance

pytestmark = pytest.mark.gpu


def _views(batch, dim, N, L, dtype, pad_rows, pad_t, share_b, seed):
    """Inputs as strided views plus their dense copies."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    dev = "cuda"

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=dev).to(dtype)

    # u and z: the two halves of one (batch, 2 dim, L + pad_t) projection
    xz = randn(batch, 2 * dim, L + pad_t)
    u, z = xz[:, :dim, :L], xz[:, dim:, :L]
    delta = randn(batch, dim + pad_rows, L + pad_t)[:, :dim, :L]
    if share_b:
        B = randn(1, N, L).expand(batch, N, L)
    else:
        B = randn(batch, N + pad_rows, L + pad_t)[:, :N, :L]
    C = randn(batch, 2 * N + pad_rows, L + pad_t)[:, N:2 * N, :L]
    A = -(torch.arange(1, N + 1, device=dev, dtype=torch.float32)
          .repeat(dim, 1) * torch.exp(0.1 * torch.randn(dim, N, generator=g, device=dev)))
    D = torch.randn(dim, generator=g, device=dev)
    v = 1e-3 + (0.1 - 1e-3) * torch.rand(dim, generator=g, device=dev)
    delta_bias = torch.log(torch.expm1(v))
    return dict(u=u, delta=delta, z=z, B=B, C=C, A=A.contiguous(), D=D,
                delta_bias=delta_bias)


CASES = [
    # name, batch, dim, N, L, dtype, pad_rows, pad_t, share_b, out_dtype, splits
    ("bf16-tma", 2, 80, 16, 1000, torch.bfloat16, 2, 8, False, torch.float32, 0),
    ("bf16-plain", 2, 80, 16, 1000, torch.bfloat16, 1, 1, False, torch.float32, 0),
    ("f32-tma", 2, 48, 16, 600, torch.float32, 3, 4, False, torch.float32, 0),
    ("f32-plain-N5", 3, 40, 5, 333, torch.float32, 1, 3, False, torch.float32, 0),
    ("bf16-shared-B", 3, 64, 16, 512, torch.bfloat16, 0, 0, True, torch.float32, 0),
    ("bf16-split", 1, 64, 16, 4000, torch.bfloat16, 2, 8, False, torch.float32, 3),
    ("bf16-y-bf16", 2, 80, 16, 1000, torch.bfloat16, 2, 8, False, torch.bfloat16, 0),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_strided_views_match_the_oracle(case):
    name, batch, dim, N, L, dtype, pad_rows, pad_t, share_b, out_dtype, splits = case
    inp = _views(batch, dim, N, L, dtype, pad_rows, pad_t, share_b, seed=4800 + len(name))
    assert not inp["u"].is_contiguous() and not inp["z"].is_contiguous()
    # y inside a larger buffer: rows padded by 4 steps, one spare channel
    ybuf = torch.full((batch, dim + 1, L + 4), float("nan"), device="cuda", dtype=out_dtype)
    y = ybuf[:, :dim, :L]
    last = torch.empty(batch, dim, N, device="cuda", dtype=torch.float32)
    sss.selective_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                           D=inp["D"], z=inp["z"], delta_bias=inp["delta_bias"],
                           y=y, last_state=last, plan_splits=splits,
                           check_status=True)
    torch.cuda.synchronize()
    # the padding of the output buffer is untouched
    assert torch.isnan(ybuf[:, dim, :].float()).all()
    assert torch.isnan(ybuf[:, :, L:].float()).all()

    w = workloads.custom(batch=batch, dim=dim, dstate=N, seqlen=L,
                         in_dtype="bf16" if dtype == torch.bfloat16 else "f32",
                         has_z=True)
    dense = {k: (v.contiguous() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    dense["h0"] = None
    y_ref, last_ref = run_oracle(w, dense, return_last_state=True)
    err = norm_err(y.float().cpu().numpy(), y_ref)
    assert err <= tolerance(w.in_dtype, out_dtype), (name, err)
    assert norm_err(last.cpu().numpy(), last_ref) <= tolerance(w.in_dtype), name


def test_strided_and_dense_runs_agree_bitwise():
    """The same values through views and through dense copies give the same
    bits: strides change addressing only, never the arithmetic."""
    inp = _views(2, 80, 16, 1024, torch.bfloat16, 2, 8, False, seed=4848)
    dense = {k: v.contiguous() for k, v in inp.items()}
    ys = []
    for src in (inp, dense):
        ys.append(sss.selective_scan_fwd(src["u"], src["delta"], src["A"], src["B"], src["C"],
                                         D=src["D"], z=src["z"], delta_bias=src["delta_bias"],
                                         check_status=True))
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1])
