"""The chunked evaluation of the Mamba-2 (SSD) scan, modelled in fp64 on the
CPU and checked against the oracle's sequential recurrence.

The CUDA kernel evaluates the scan chunk by chunk as four matrix products
(scores C B^T, the masked product with X, the readout of the carried state,
the chunk's state update), with the decay between steps s <= t factored
into a per-row and a per-column factor per 32-step block, and the diagonal
blocks factored the same way unless a block decays by 2^64 or more.  This
model follows the same decomposition in numpy:

* without rounding it must equal the recurrence to fp64 rounding, which
  pins the algebra of the decomposition (the masks, the factored decays,
  the carried state and its decay) independently of the GPU;
* with the kernel's three bf16 roundings (masked scores, weighted inputs,
  carried state copy) it must stay inside the tolerance the GPU parity
  tests use, one unit of bf16 roundoff (2^-8, rounded up to 4e-3) of
  max |y|, which pins that bound's derivation.

Test infrastructure only; it shares nothing with the CUDA code.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

Q = 128
LOG2E = 1.4426950408889634
U_BF16 = 2.0 ** -8


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()


def _softplus(v):
    return np.logaddexp(0.0, v)


def chunked_ssd(x, dt, A, B, C, D, z, dt_bias, h0, rounding):
    """y, last_state of the SSD scan evaluated the way the kernel does."""
    bt, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    rd = _bf16 if rounding else (lambda a: a)
    y = np.zeros_like(x)
    last = np.zeros((bt, H, P, N))
    nch = -(-L // Q)
    for b in range(bt):
        for h in range(H):
            g = h // (H // G)
            state = np.zeros((N, P)) if h0 is None else h0[b, h].T.copy()  # [n][p]
            for c in range(nch):
                t0, t1 = c * Q, min(L, (c + 1) * Q)
                n = t1 - t0
                Xc = np.zeros((Q, P))
                Xc[:n] = x[b, t0:t1, h]
                Bc = np.zeros((Q, N))
                Bc[:n] = B[b, t0:t1, g]
                Cc = np.zeros((Q, N))
                Cc[:n] = C[b, t0:t1, g]
                step = np.zeros(Q)
                step[:n] = _softplus(dt[b, t0:t1, h] + (dt_bias[h] if dt_bias is not None else 0.0))
                cum = np.cumsum(step * A[h] * LOG2E)
                cl = cum[-1]
                # per-column factors 2^(c_end - c_s) Delta_s, c_end the last
                # step of s's 32-step block
                cend = np.repeat(cum[31::32], 32)
                colf = np.exp2(cend - cum) * step
                S = Cc @ Bc.T
                Sp = np.zeros((Q, Q))
                for tb in range(4):
                    rows = slice(32 * tb, 32 * tb + 32)
                    for gb in range(tb + 1):
                        cols = slice(32 * gb, 32 * gb + 32)
                        rf = np.exp2(cum[rows] - cum[32 * gb + 31])[:, None]
                        if gb < tb:
                            Sp[rows, cols] = S[rows, cols] * rf * colf[cols][None, :]
                        else:
                            if cum[32 * gb] - cum[32 * gb + 31] < 64.0:
                                blk = S[rows, cols] * rf * colf[cols][None, :]
                            else:
                                blk = (S[rows, cols] *
                                       np.exp2(cum[rows][:, None] - cum[cols][None, :]) *
                                       step[cols][None, :])
                            Sp[rows, cols] = np.tril(blk)
                Yd = rd(Sp) @ Xc
                YO = Cc @ rd(state)
                yc = Yd + np.exp2(cum)[:, None] * YO
                if D is not None:
                    yc += D[h] * Xc
                if z is not None:
                    zc = np.zeros((Q, P))
                    zc[:n] = z[b, t0:t1, h]
                    yc *= zc / (1.0 + np.exp(-zc))
                y[b, t0:t1, h] = yc[:n]
                Xpp = Xc * (step * np.exp2(cl - cum))[:, None]
                state = np.exp2(cl) * state + Bc.T @ rd(Xpp)
            last[b, h] = state.T
    return y, last


def _case(name, batch, L, H, G, has_z, h0, seed, bias_shift=0.0):
    w = workloads.SsdWorkload(name, batch, L, H, ngroups=G, has_z=has_z)
    inp = workloads.make_ssd_inputs(w, seed=seed, h0=h0)
    if bias_shift:
        inp["dt_bias"] = inp["dt_bias"] + bias_shift
    return workloads.to_numpy_f64(inp)


CASES = [
    # name, batch, L, heads, groups, z, h0, dt_bias shift
    ("ragged-two-groups", 2, 300, 4, 2, True, True, 0.0),
    ("one-short-chunk", 1, 50, 2, 1, False, False, 0.0),
    ("long-carry", 1, 1000, 2, 1, True, True, 0.0),
    # steps near 2-7: blocks decay by more than 2^64, the unfactored path
    ("strong-decay", 1, 400, 2, 1, False, True, 6.0),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_chunked_decomposition_is_the_recurrence(case):
    name, batch, L, H, G, has_z, h0, shift = case
    h = _case(name, batch, L, H, G, has_z, h0, 7700 + L, shift)
    args = (h["x"], h["dt"], h["A"], h["B"], h["C"], h["D"], h["z"], h["dt_bias"], h["h0"])
    y_ref, last_ref = oracle.ssd_scan(*args[:5], D=h["D"], z=h["z"], dt_bias=h["dt_bias"],
                                      h0=h["h0"], return_last_state=True)
    y, last = chunked_ssd(*args, rounding=False)
    assert np.abs(y - y_ref).max() <= 1e-10 * np.abs(y_ref).max()
    assert np.abs(last - last_ref).max() <= 1e-10 * max(np.abs(last_ref).max(), 1e-300)
    if shift:
        # the case does reach the unfactored diagonal path
        step = _softplus(h["dt"][0, :, 0] + h["dt_bias"][0])
        cum = np.cumsum(step * h["A"][0] * LOG2E)
        assert (cum[:-32:32] - cum[31::32]).max() >= 64.0


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_bf16_operands_stay_inside_the_parity_tolerance(case):
    name, batch, L, H, G, has_z, h0, shift = case
    h = _case(name, batch, L, H, G, has_z, h0, 7700 + L, shift)
    args = (h["x"], h["dt"], h["A"], h["B"], h["C"], h["D"], h["z"], h["dt_bias"], h["h0"])
    y_ref, last_ref = oracle.ssd_scan(*args[:5], D=h["D"], z=h["z"], dt_bias=h["dt_bias"],
                                      h0=h["h0"], return_last_state=True)
    y, last = chunked_ssd(*args, rounding=True)
    err = np.abs(y - y_ref).max() / np.abs(y_ref).max()
    err_last = np.abs(last - last_ref).max() / np.abs(last_ref).max()
    assert err <= 4e-3, err
    assert err_last <= 4e-3, err_last
    # and the roundings are visible at all (the model does round)
    assert err > 1e-6
