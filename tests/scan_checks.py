"""Shared helpers of the GPU parity tests: run the CUDA path and the fp64
oracle on the same seeded inputs and compare.

Tolerances (max |y_gpu - y_oracle| / max |y_oracle|, the oracle fed the
very values the GPU reads, i.e. after bf16 rounding):
  fp32 inputs, fp32 y   1e-4
  bf16 inputs, fp32 y   2e-3
  bf16 y                2e-3 + 2^-8 (rounding y itself to bf16 costs up to
                        2^-8 relative)
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import selective_state_space_48_b200 as sss
import workloads

TOL_F32 = 1e-4
TOL_BF16 = 2e-3
TOL_BF16_OUT = 2e-3 + 2.0 ** -8


def tolerance(in_dtype: str, out_dtype=torch.float32) -> float:
    if out_dtype == torch.bfloat16:
        return TOL_BF16_OUT
    return TOL_F32 if in_dtype == "f32" else TOL_BF16


def norm_err(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    scale = np.abs(want).max()
    if scale == 0:
        return float(np.abs(got).max())
    return float(np.abs(got - want).max() / scale)


def gpu_inputs(w, seed=None, h0=False):
    inp = workloads.make_inputs(w, seed=seed, device="cuda")
    if h0:
        g = torch.Generator(device="cuda")
        g.manual_seed(12345 if seed is None else seed + 1)
        inp["h0"] = torch.randn(w.batch, w.dim, w.dstate, generator=g,
                                device="cuda", dtype=torch.float32)
    else:
        inp["h0"] = None
    return inp


def run_gpu(w, inp, out_dtype=torch.float32, plan_splits=0,
            return_last_state=False, **kw):
    return sss.selective_scan_fwd(
        inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
        z=inp["z"], delta_bias=inp["delta_bias"], delta_softplus=w.softplus,
        h0=inp["h0"], return_last_state=return_last_state,
        out_dtype=out_dtype, plan_splits=plan_splits, **kw)


def run_oracle(w, inp, return_last_state=False):
    h = workloads.to_numpy_f64(inp)
    return oracle.selective_scan(
        h["u"], h["delta"], h["A"], h["B"], h["C"], D=h["D"], z=h["z"],
        delta_bias=h["delta_bias"], delta_softplus=w.softplus, h0=h["h0"],
        return_last_state=return_last_state)


def sampled_channels(w, count=24, seed=0):
    """(b, d) pairs spread over the tensor: first, last, tile edges, random."""
    rng = np.random.default_rng(seed)
    picks = {(0, 0), (w.batch - 1, w.dim - 1)}
    for d in (31, 32, 63, 64):
        if d < w.dim:
            picks.add((0, d))
    while len(picks) < min(count, w.batch * w.dim):
        picks.add((int(rng.integers(w.batch)), int(rng.integers(w.dim))))
    return sorted(picks)


def oracle_on_channels(w, inp, picks):
    """Run the oracle only on the sampled channels (full length)."""
    out = {}
    for b, d in picks:
        sl = lambda t: None if t is None else t[b:b + 1, d:d + 1].detach().cpu().double().numpy()
        bc = lambda t: t[b:b + 1].detach().cpu().double().numpy()
        pd = lambda t: None if t is None else t[d:d + 1].detach().cpu().double().numpy()
        h0 = inp.get("h0")
        y = oracle.selective_scan(
            sl(inp["u"]), sl(inp["delta"]), pd(inp["A"]), bc(inp["B"]),
            bc(inp["C"]), D=pd(inp["D"]), z=sl(inp["z"]),
            delta_bias=pd(inp["delta_bias"]), delta_softplus=w.softplus,
            h0=None if h0 is None else h0[b:b + 1, d:d + 1].cpu().double().numpy())
        out[(b, d)] = y[0, 0]
    return out
