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
from oracle.compare import ErrorStats
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


# ---------------------------------------------------------------- full size
#
# Full-size workloads are compared element by element: the oracle runs on
# every channel, a block of channels of one batch row at a time (so host
# memory stays bounded), and each block of the GPU output is compared with
# it.  The error is normalised by the largest |y_oracle| over the whole
# output, as everywhere else.


def _rows(t, b, d0, d1):
    return None if t is None else t[b:b + 1, d0:d1].detach().float().cpu().double().numpy()


def _chan(t, d0, d1):
    return None if t is None else t[d0:d1].detach().float().cpu().double().numpy()


def oracle_blocks(w, inp, block=512, cu_seqlens=None, trapezoid=False):
    """(b, d0, d1, y_oracle[1, d1-d0, L]) for every block of channels of
    every batch row, in order."""
    h0 = inp.get("h0")
    for b in range(w.batch):
        Bh = inp["B"][b:b + 1].detach().float().cpu().double().numpy()
        Ch = inp["C"][b:b + 1].detach().float().cpu().double().numpy()
        for d0 in range(0, w.dim, block):
            d1 = min(w.dim, d0 + block)
            y = oracle.selective_scan(
                _rows(inp["u"], b, d0, d1), _rows(inp["delta"], b, d0, d1),
                _chan(inp["A"], d0, d1), Bh, Ch, D=_chan(inp["D"], d0, d1),
                z=_rows(inp["z"], b, d0, d1), delta_bias=_chan(inp["delta_bias"], d0, d1),
                delta_softplus=w.softplus, h0=_rows(h0, b, d0, d1),
                cu_seqlens=cu_seqlens, trapezoid=trapezoid)
            yield b, d0, d1, y


def compare_all_channels(w, inp, y, block=512, cu_seqlens=None, trapezoid=False):
    """ErrorStats of the GPU output y (batch, dim, L) against the oracle on
    every element."""
    st = ErrorStats()
    for b, d0, d1, want in oracle_blocks(w, inp, block, cu_seqlens, trapezoid):
        got = y[b:b + 1, d0:d1].detach().float().cpu().double().numpy()
        st.add(got, want)
    return st
