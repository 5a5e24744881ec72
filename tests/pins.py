"""Pins of the fp64 oracle against facts it does not compute itself.

Each ``pin_*`` function takes a loaded oracle library handle and raises
AssertionError when the oracle disagrees with:
  * the worked example printed on the pages (tests/golden/),
  * closed forms (brute-force unrolled sums in mpmath, the sigmoid-product
    form of the N=1 gate, the LTI convolution computed with numpy.convolve),
  * limits and special cases (Delta -> 0, Delta large, B = 0, z = 0).
None of them re-uses the oracle's own recurrence.  ``test_oracle_pins.py``
runs them on the oracle; ``test_oracle_planted_mistakes.py`` runs them on
deliberately broken copies of the oracle to show each plausible mistake is
caught by at least one pin.
"""
from __future__ import annotations

import math
import os

import mpmath
import numpy as np
import scipy.special

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_golden(name: str) -> dict:
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            k, v = (s.strip() for s in line.split("=", 1))
            vals[k] = float(v)
    return vals


def _rng(seed):
    return np.random.default_rng(seed)


def _close(got, want, rtol, atol=0.0, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    bound = atol + rtol * np.abs(want)
    assert np.all(err <= bound), (
        f"{what}: max err {err.max():.3e} (bound {bound.max():.3e})")


# --------------------------------------------------------------------------
# "The relay": the page's worked example, through combine and through the
# scan itself.


def pin_combine_worked_example(lib):
    g = load_golden("relay_worked_example.txt")
    a, b = oracle.combine(g["a1"], g["b1"], g["a2"], g["b2"], lib=lib)
    _close([a, b], [g["a12"], g["b12"]], 1e-15, 1e-15, "combine example")


def _worked_example_inputs(g, x0):
    """N=1, one channel, two steps with (a, b) = (0.6, 0.4) then (0.5, 1.0),
    realised with softplus off, delta_bias = 0, C = 1, D = 0 and inputs
    u = (2, -0.5), B chosen so that delta * B * u = b."""
    A_val = math.log(g["a1"])               # delta_1 = 1 -> exp(A) = 0.6
    d2 = math.log(g["a2"]) / A_val          # exp(d2 * A) = 0.5
    delta = np.array([[[1.0, d2]]])
    u = np.array([[[2.0, -0.5]]])
    B = np.array([[[g["b1"] / (1.0 * 2.0), g["b2"] / (d2 * -0.5)]]])
    C = np.ones((1, 1, 2))
    A = np.array([[A_val]])
    h0 = np.array([[[x0]]])
    return u, delta, A, B, C, h0


def pin_scan_worked_example(lib):
    g = load_golden("relay_worked_example.txt")
    for x0 in (0.0, 2.5, -7.0):
        u, delta, A, B, C, h0 = _worked_example_inputs(g, x0)
        y, last = oracle.selective_scan(u, delta, A, B, C, D=None, z=None,
                                        delta_bias=None, delta_softplus=False,
                                        h0=h0, return_last_state=True, lib=lib)
        want = [g["after_step1_fade"] * x0 + g["after_step1_add"],
                g["a12"] * x0 + g["b12"]]
        _close(y[0, 0], want, 1e-14, 1e-14, "scan realises the relay example")
        _close(last[0, 0, 0], want[1], 1e-14, 1e-14, "last state")


def pin_state_update_worked_example(lib):
    g = load_golden("relay_worked_example.txt")
    x0 = 1.75
    u, delta, A, B, C, h0 = _worked_example_inputs(g, x0)
    st = h0.copy()
    outs = []
    for t in range(2):
        st, y = oracle.selective_state_update(
            st, u[:, :, t], delta[:, :, t], A, B[:, :, t], C[:, :, t],
            D=None, z=None, dt_bias=None, dt_softplus=False, lib=lib)
        outs.append(y[0, 0])
    want = [0.6 * x0 + 0.4, 0.3 * x0 + 1.2]
    _close(outs, want, 1e-14, 1e-14, "state update realises the example")
    _close(st[0, 0, 0], want[1], 1e-14, 1e-14, "state after two steps")


def pin_state_update_special_cases(lib):
    """B = 0 leaves D x silu(z) and the state faded by exp(Delta A); z = 0
    closes the gate."""
    rng = _rng(19)
    batch, dim, N = 2, 3, 4
    st = rng.normal(size=(batch, dim, N))
    x = rng.normal(size=(batch, dim))
    dt = rng.normal(size=(batch, dim))
    A = -rng.uniform(0.5, 2.0, size=(dim, N))
    C = rng.normal(size=(batch, N))
    D = rng.normal(size=dim)
    z = rng.normal(size=(batch, dim))
    bias = rng.normal(size=dim)
    new, y = oracle.selective_state_update(st, x, dt, A, np.zeros((batch, N)),
                                           np.zeros((batch, N)), D=D, z=z,
                                           dt_bias=bias, lib=lib)
    _close(y, D[None, :] * x * z * scipy.special.expit(z), 1e-14, 1e-15,
           "update with B = C = 0")
    # softplus(v) = -log(sigmoid(-v)), so exp(Delta A) = sigmoid(-v) ** (-A)
    v = dt + bias[None, :]
    fade = scipy.special.expit(-v)[:, :, None] ** (-A[None, :, :])
    _close(new, fade * st, 1e-13, 1e-15, "state fades by exp(Delta A)")
    _, y0 = oracle.selective_state_update(st, x, dt, A, rng.normal(size=(batch, N)),
                                          C, D=D, z=np.zeros_like(z),
                                          dt_bias=bias, lib=lib)
    assert np.all(y0 == 0.0)


# --------------------------------------------------------------------------
# Associativity (same section): any grouping of the steps gives the same map.


def pin_combine_associative(lib):
    rng = _rng(11)
    for trial in range(20):
        L = int(rng.integers(2, 40))
        a = rng.uniform(0.0, 1.0, L)
        b = rng.normal(size=L)
        h = rng.normal()
        # the steps applied one after another: the meaning of the pairs
        seq = h
        for t in range(L):
            seq = a[t] * seq + b[t]
        # random binary tree over the same steps
        items = [(a[t], b[t]) for t in range(L)]
        while len(items) > 1:
            i = int(rng.integers(0, len(items) - 1))
            p, q = items[i], items[i + 1]
            items[i:i + 2] = [oracle.combine(p[0], p[1], q[0], q[1], lib=lib)]
        A_, B_ = items[0]
        _close(A_ * h + B_, seq, 1e-12, 1e-12, "random grouping")


# --------------------------------------------------------------------------
# Closed form: unroll the recurrence into explicit sums, in mpmath.


def _mp_softplus(x):
    return mpmath.log1p(mpmath.e ** x)


def _mp_silu(z):
    return z / (1 + mpmath.e ** (-z))


def _brute_force(u, delta, A, B, C, D, z, bias, softplus, h0):
    """h_t[n] = exp(A[n] * sum_{r<=t} Dt_r) h0[n]
              + sum_{s<=t} exp(A[n] * sum_{r=s+1..t} Dt_r) Dt_s B_s[n] u_s
       y_t    = (sum_n C_t[n] h_t[n] + D u_t) * silu(z_t)."""
    mpmath.mp.dps = 40
    batch, dim, L = u.shape
    N = A.shape[1]
    y = np.zeros((batch, dim, L))
    last = np.zeros((batch, dim, N))
    for b in range(batch):
        for d in range(dim):
            x = [mpmath.mpf(float(delta[b, d, t])) +
                 (mpmath.mpf(float(bias[d])) if bias is not None else 0)
                 for t in range(L)]
            dt = [_mp_softplus(v) if softplus else v for v in x]
            pref = [mpmath.mpf(0)]
            for t in range(L):
                pref.append(pref[-1] + dt[t])
            for t in range(L):
                acc = mpmath.mpf(0)
                for n in range(N):
                    a = mpmath.mpf(float(A[d, n]))
                    h = mpmath.mpf(0)
                    if h0 is not None:
                        h += mpmath.e ** (a * pref[t + 1]) * float(h0[b, d, n])
                    for s in range(t + 1):
                        h += (mpmath.e ** (a * (pref[t + 1] - pref[s + 1])) *
                              dt[s] * float(B[b, n, s]) * float(u[b, d, s]))
                    acc += float(C[b, n, t]) * h
                    if t == L - 1:
                        last[b, d, n] = float(h)
                yt = acc + (float(D[d]) if D is not None else 0) * float(u[b, d, t])
                if z is not None:
                    yt *= _mp_silu(mpmath.mpf(float(z[b, d, t])))
                y[b, d, t] = float(yt)
    return y, last


def pin_brute_force_unrolled(lib):
    rng = _rng(3)
    cases = [
        dict(batch=1, dim=2, N=3, L=9, z=True, D=True, bias=True, sp=True, h0=True),
        dict(batch=2, dim=1, N=2, L=12, z=False, D=True, bias=False, sp=True, h0=False),
        dict(batch=1, dim=1, N=4, L=7, z=True, D=False, bias=True, sp=False, h0=True),
    ]
    for c in cases:
        bt, dm, N, L = c["batch"], c["dim"], c["N"], c["L"]
        u = rng.normal(size=(bt, dm, L))
        if c["sp"]:
            delta = rng.normal(size=(bt, dm, L))
        else:
            delta = rng.uniform(0.05, 0.6, size=(bt, dm, L))
        A = -rng.uniform(0.2, 3.0, size=(dm, N))
        B = rng.normal(size=(bt, N, L))
        C = rng.normal(size=(bt, N, L))
        D = rng.normal(size=dm) if c["D"] else None
        z = rng.normal(size=(bt, dm, L)) if c["z"] else None
        bias = rng.normal(size=dm) * 0.5 if c["bias"] else None
        h0 = rng.normal(size=(bt, dm, N)) if c["h0"] else None
        want, want_last = _brute_force(u, delta, A, B, C, D, z, bias, c["sp"], h0)
        got, got_last = oracle.selective_scan(
            u, delta, A, B, C, D=D, z=z, delta_bias=bias,
            delta_softplus=c["sp"], h0=h0, return_last_state=True, lib=lib)
        _close(got, want, 1e-11, 1e-12, f"brute force {c}")
        _close(got_last, want_last, 1e-11, 1e-12, f"brute force last {c}")


# --------------------------------------------------------------------------
# "From Convolutions to State Spaces: S4" / "S4: The Same Operation, Two
# Faces": with Delta, B, C fixed over t the scan is the causal convolution
# y = K * u + D u with K_k = sum_n C[n] exp(k Delta A[n]) Delta B[n].


def pin_lti_convolution(lib):
    rng = _rng(5)
    for trial in range(4):
        dim, N, L = 3, int(rng.integers(1, 6)), int(rng.integers(20, 90))
        u = rng.normal(size=(1, dim, L))
        dconst = rng.normal(size=dim)
        delta = np.repeat(dconst[None, :, None], L, axis=2)
        Bc = rng.normal(size=N)
        Cc = rng.normal(size=N)
        B = np.repeat(Bc[None, :, None], L, axis=2)
        C = np.repeat(Cc[None, :, None], L, axis=2)
        A = -rng.uniform(0.05, 2.0, size=(dim, N))
        D = rng.normal(size=dim)
        y = oracle.selective_scan(u, delta, A, B, C, D=D, z=None,
                                  delta_bias=None, delta_softplus=True, lib=lib)
        for d in range(dim):
            step = float(scipy.special.softplus(dconst[d])) if hasattr(
                scipy.special, "softplus") else math.log1p(math.exp(dconst[d]))
            k = np.arange(L)
            K = (Cc[None, :] * np.exp(np.outer(k, step * A[d])) *
                 (step * Bc)[None, :]).sum(axis=1)
            conv = np.convolve(u[0, d], K)[:L] + D[d] * u[0, d]
            _close(y[0, d], conv, 1e-11, 1e-11, "LTI convolution")


# --------------------------------------------------------------------------
# "What selective changed": with one state the update is a gate.  With
# A = -1 and Delta = softplus(x), exp(Delta A) = 1 / (1 + e^x) = sigmoid(-x),
# so with no input (B = 0) and C = 1, y_t = h0 * prod_{r<=t} sigmoid(-x_r).


def pin_n1_gate(lib):
    rng = _rng(7)
    L = 50
    x = rng.normal(size=L) * 2.0
    bias = 0.3
    u = rng.normal(size=(1, 1, L))
    y = oracle.selective_scan(u, (x - bias)[None, None, :], np.array([[-1.0]]),
                              np.zeros((1, 1, L)), np.ones((1, 1, L)),
                              D=None, z=None, delta_bias=np.array([bias]),
                              delta_softplus=True, h0=np.array([[[1.5]]]),
                              lib=lib)
    want = 1.5 * np.cumprod(scipy.special.expit(-x))
    _close(y[0, 0], want, 1e-13, 1e-15, "N=1 gate closed form")
    # with input: h_t = sigmoid(-x_t) h_{t-1} + softplus(x_t) B_t u_t
    B = rng.normal(size=(1, 1, L))
    y2 = oracle.selective_scan(u, (x - bias)[None, None, :], np.array([[-1.0]]),
                               B, np.ones((1, 1, L)), D=None, z=None,
                               delta_bias=np.array([bias]), delta_softplus=True,
                               h0=None, lib=lib)
    g = scipy.special.expit(-x)
    sp = -np.log(g)                     # softplus(x) = -log(sigmoid(-x))
    want2 = np.zeros(L)
    for t in range(L):
        want2[t] = sum(np.prod(g[s + 1:t + 1]) * sp[s] * B[0, 0, s] * u[0, 0, s]
                       for s in range(t + 1))
    _close(y2[0, 0], want2, 1e-12, 1e-13, "N=1 gate with input")


# --------------------------------------------------------------------------
# Delta limits ("The Solution and Its Price"; "The Selection Mechanism"):
# Delta -> 0 leaves the state untouched and ignores the token; a large Delta
# overwrites the state with the current input.


def pin_delta_limits(lib):
    rng = _rng(9)
    dim, N, L = 2, 3, 10
    u = rng.normal(size=(1, dim, L))
    A = -rng.uniform(0.5, 2.0, size=(dim, N))
    B = rng.normal(size=(1, N, L))
    C = rng.normal(size=(1, N, L))
    D = rng.normal(size=dim)
    h0 = rng.normal(size=(1, dim, N))
    # tiny step: softplus(-60) ~ 8.8e-27
    y = oracle.selective_scan(u, np.full((1, dim, L), -60.0), A, B, C, D=D,
                              delta_softplus=True, h0=h0, lib=lib)
    want = np.einsum("nt,dn->dt", C[0], h0[0]) + D[:, None] * u[0]
    _close(y[0], want, 1e-12, 1e-14, "Delta -> 0 keeps the state")
    # large step: softplus(60) = 60, exp(60 A) < 1e-13 -> h_t = 60 B_t u_t
    y = oracle.selective_scan(u, np.full((1, dim, L), 60.0), A, B, C, D=D,
                              delta_softplus=True, h0=h0, lib=lib)
    h = 60.0 * B[0][None, :, :] * u[0][:, None, :]          # (dim, N, L)
    want = np.einsum("nt,dnt->dt", C[0], h) + D[:, None] * u[0]
    _close(y[0], want, 1e-10, 1e-10, "large Delta overwrites the state")


# --------------------------------------------------------------------------
# Special cases of the gate, the skip term and the step size.


def pin_special_cases(lib):
    rng = _rng(13)
    dim, N, L = 3, 4, 16
    u = rng.normal(size=(2, dim, L))
    delta = rng.normal(size=(2, dim, L))
    A = -rng.uniform(0.5, 2.0, size=(dim, N))
    B = rng.normal(size=(2, N, L))
    C = rng.normal(size=(2, N, L))
    D = rng.normal(size=dim)
    z = rng.normal(size=(2, dim, L))
    # z = 0 closes the gate completely
    y = oracle.selective_scan(u, delta, A, B, C, D=D, z=np.zeros_like(z), lib=lib)
    assert np.all(y == 0.0), "silu(0) gate must give y = 0"
    # B = 0: only the skip term survives, gated by silu(z)
    y = oracle.selective_scan(u, delta, A, np.zeros_like(B), C, D=D, z=z, lib=lib)
    want = D[None, :, None] * u * z * scipy.special.expit(z)
    _close(y, want, 1e-14, 1e-15, "B = 0 leaves D u silu(z)")
    # softplus off with delta = 1/|A|: each step fades by exactly e^-1
    Aone = np.array([[-2.0]])
    y = oracle.selective_scan(np.ones((1, 1, 5)), np.full((1, 1, 5), 0.5), Aone,
                              np.zeros((1, 1, 5)), np.ones((1, 1, 5)),
                              delta_softplus=False, h0=np.array([[[1.0]]]),
                              lib=lib)
    _close(y[0, 0], np.exp(-np.arange(1, 6)), 1e-15, 0.0, "fade e^-1 per step")


def pin_softplus_silu(lib):
    for x in (-745.0, -40.0, -5.0, -0.5, 0.0, 1e-8, 0.5, 5.0, 40.0, 700.0):
        want = float(_mp_softplus(mpmath.mpf(x)))
        got = oracle.softplus(x, lib=lib)
        assert abs(got - want) <= 2e-16 * abs(want) + 1e-320, (x, got, want)
        wz = float(_mp_silu(mpmath.mpf(x))) if x > -700 else 0.0
        gz = oracle.silu(x, lib=lib)
        assert abs(gz - wz) <= 4e-16 * abs(wz) + 1e-300, (x, gz, wz)


# --------------------------------------------------------------------------
# Scan-then-resume: the state hands over exactly between two calls.


def pin_resume(lib):
    rng = _rng(17)
    dim, N, L = 2, 3, 30
    args = dict(u=rng.normal(size=(1, dim, L)), delta=rng.normal(size=(1, dim, L)),
                B=rng.normal(size=(1, N, L)), C=rng.normal(size=(1, N, L)),
                z=rng.normal(size=(1, dim, L)))
    A = -rng.uniform(0.1, 2.0, size=(dim, N))
    D = rng.normal(size=dim)
    bias = rng.normal(size=dim)
    y, last = oracle.selective_scan(args["u"], args["delta"], A, args["B"],
                                    args["C"], D=D, z=args["z"], delta_bias=bias,
                                    return_last_state=True, lib=lib)
    cut = 13
    p1 = {k: v[..., :cut] for k, v in args.items()}
    p2 = {k: v[..., cut:] for k, v in args.items()}
    y1, s1 = oracle.selective_scan(p1["u"], p1["delta"], A, p1["B"], p1["C"],
                                   D=D, z=p1["z"], delta_bias=bias,
                                   return_last_state=True, lib=lib)
    y2, s2 = oracle.selective_scan(p2["u"], p2["delta"], A, p2["B"], p2["C"],
                                   D=D, z=p2["z"], delta_bias=bias, h0=s1,
                                   return_last_state=True, lib=lib)
    _close(np.concatenate([y1, y2], axis=-1), y, 1e-14, 1e-14, "resume y")
    _close(s2, last, 1e-14, 1e-14, "resume state")


# --------------------------------------------------------------------------
# Packed sequences: a row holding several independent sequences (offsets
# cu_seqlens) is the concatenation of their separate scans, each from an
# empty state except the first, which starts from h0.  Checked against the
# mpmath unrolled sums of every sequence on its own, so the reset logic is
# pinned to the closed form, not to the oracle's recurrence.


def pin_packed_sequences(lib):
    rng = _rng(23)
    bt, dm, N, L = 2, 2, 3, 11
    # a 1-step sequence, an empty one, interior starts inside and at the end
    cu = [0, 1, 5, 5, 9, 11]
    u = rng.normal(size=(bt, dm, L))
    delta = rng.normal(size=(bt, dm, L))
    A = -rng.uniform(0.2, 2.0, size=(dm, N))
    B = rng.normal(size=(bt, N, L))
    C = rng.normal(size=(bt, N, L))
    D = rng.normal(size=dm)
    z = rng.normal(size=(bt, dm, L))
    bias = rng.normal(size=dm) * 0.5
    h0 = rng.normal(size=(bt, dm, N))
    want = np.zeros((bt, dm, L))
    want_last = None
    for i in range(len(cu) - 1):
        a, b = cu[i], cu[i + 1]
        if a == b:
            continue
        sl = slice(a, b)
        yi, li = _brute_force(u[..., sl], delta[..., sl], A, B[..., sl], C[..., sl],
                              D, z[..., sl], bias, True, h0 if i == 0 else None)
        want[..., sl] = yi
        want_last = li
    got, got_last = oracle.selective_scan(u, delta, A, B, C, D=D, z=z, delta_bias=bias,
                                          h0=h0, return_last_state=True, lib=lib,
                                          cu_seqlens=cu)
    _close(got, want, 1e-11, 1e-12, "packed sequences y")
    _close(got_last, want_last, 1e-11, 1e-12, "packed sequences last state")
    # one sequence spanning the row is the plain scan
    plain = oracle.selective_scan(u, delta, A, B, C, D=D, z=z, delta_bias=bias,
                                  h0=h0, lib=lib)
    one = oracle.selective_scan(u, delta, A, B, C, D=D, z=z, delta_bias=bias,
                                h0=h0, lib=lib, cu_seqlens=[0, L])
    _close(one, plain, 0.0, 0.0, "one packed sequence")


# --------------------------------------------------------------------------
# The backward pass: every gradient against central finite differences of
# the forward oracle (pinned above) along a random direction, i.e.
# <grad_X, V> = (F(X + eps V) - F(X - eps V)) / (2 eps) with
# F = sum(dy * y) + sum(d_last * last_state).


def _fd_check(lib, case, seed):
    rng = _rng(seed)
    bt, dm, N, L = case["shape"]
    sp = case["softplus"]
    X = dict(
        u=rng.normal(size=(bt, dm, L)),
        delta=rng.normal(size=(bt, dm, L)) if sp else rng.uniform(0.05, 0.6, size=(bt, dm, L)),
        A=-rng.uniform(0.2, 2.0, size=(dm, N)),
        B=rng.normal(size=(bt, N, L)), C=rng.normal(size=(bt, N, L)),
        D=rng.normal(size=dm), z=rng.normal(size=(bt, dm, L)),
        delta_bias=rng.normal(size=dm) * 0.5, h0=rng.normal(size=(bt, dm, N)))
    dy = rng.normal(size=(bt, dm, L))
    d_last = rng.normal(size=(bt, dm, N))

    cu = case.get("cu")

    def F(X):
        y, last = oracle.selective_scan(X["u"], X["delta"], X["A"], X["B"], X["C"],
                                        D=X["D"], z=X["z"], delta_bias=X["delta_bias"],
                                        delta_softplus=sp, h0=X["h0"],
                                        return_last_state=True, lib=lib, cu_seqlens=cu)
        return float(np.sum(dy * y) + np.sum(d_last * last))

    g = oracle.selective_scan_bwd(X["u"], X["delta"], X["A"], X["B"], X["C"], dy,
                                  D=X["D"], z=X["z"], delta_bias=X["delta_bias"],
                                  delta_softplus=sp, h0=X["h0"], d_last=d_last, lib=lib,
                                  cu_seqlens=cu)
    names = {"u": "du", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC",
             "D": "dD", "z": "dz", "delta_bias": "ddelta_bias", "h0": "dh0"}
    eps = 1e-6
    for k, gk in names.items():
        V = rng.normal(size=X[k].shape)
        Xp = dict(X); Xp[k] = X[k] + eps * V
        Xm = dict(X); Xm[k] = X[k] - eps * V
        fd = (F(Xp) - F(Xm)) / (2 * eps)
        an = float(np.sum(g[gk] * V))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (k, fd, an, case)


def pin_backward_finite_differences(lib):
    _fd_check(lib, dict(shape=(2, 3, 4, 9), softplus=True), 31)
    _fd_check(lib, dict(shape=(1, 2, 3, 13), softplus=False), 32)
    # packed sequences (the forward oracle's packing, pinned above): starts
    # at steps 1, 5 and 6 (a one-step sequence) of 13
    _fd_check(lib, dict(shape=(2, 2, 3, 13), softplus=True, cu=[0, 1, 5, 6, 13]), 33)


# --------------------------------------------------------------------------
# "The State That Must Remember Everything", Part 7 (Mamba-3): the update
# gains a third term, the previous input.  Read as the trapezoidal rule for
# dh/dt = A h + B x: two facts pin it without re-using the recurrence.
#  * With A = 0 the state is the trapezoidal sum of B x: a cumulative sum.
#  * Against the exact solution of dh/dt = A h + sin(t), h(0) = 0, the
#    error at a fixed time falls 4x when the step halves (second order),
#    where the Euler update only halves it.


def pin_trapezoid_no_decay(lib):
    rng = _rng(41)
    bt, dm, N, L = 1, 2, 3, 17
    u = rng.normal(size=(bt, dm, L))
    delta = rng.uniform(0.05, 0.5, size=(bt, dm, L))
    A = np.zeros((dm, N))
    B = rng.normal(size=(bt, N, L))
    C = rng.normal(size=(bt, N, L))
    D = rng.normal(size=dm)
    h0 = rng.normal(size=(bt, dm, N))
    got, last = oracle.selective_scan(u, delta, A, B, C, D=D, delta_softplus=False,
                                      h0=h0, return_last_state=True, lib=lib,
                                      trapezoid=True)
    for d in range(dm):
        w = B[0] * u[0, d][None, :]                           # (N, L)
        wprev = np.concatenate([np.zeros((N, 1)), w[:, :-1]], axis=1)
        h = h0[0, d][:, None] + np.cumsum(0.5 * delta[0, d][None, :] * (wprev + w), axis=1)
        want = np.sum(C[0] * h, axis=0) + D[d] * u[0, d]
        _close(got[0, d], want, 1e-12, 1e-12, "trapezoid without decay")
        _close(last[0, d], h[:, -1], 1e-12, 1e-12, "trapezoid last state")


def _ode_error(lib, dt, trapezoid, a=-0.7, T=5.0):
    L = int(round(T / dt)) + 1
    t = np.arange(L) * dt
    u = np.sin(t)[None, None, :]
    delta = np.full((1, 1, L), dt)
    y = oracle.selective_scan(u, delta, np.array([[a]]), np.ones((1, 1, L)),
                              np.ones((1, 1, L)), delta_softplus=False, lib=lib,
                              trapezoid=trapezoid)
    exact = (-a * np.sin(T) - np.cos(T) + np.exp(a * T)) / (a * a + 1.0)
    return abs(y[0, 0, -1] - exact)


def pin_trapezoid_second_order(lib):
    e1, e2 = _ode_error(lib, 0.02, True), _ode_error(lib, 0.01, True)
    assert 3.6 < e1 / e2 < 4.4, ("trapezoid order", e1, e2)
    f1, f2 = _ode_error(lib, 0.02, False), _ode_error(lib, 0.01, False)
    assert 1.7 < f1 / f2 < 2.3, ("Euler order", f1, f2)
    assert e2 < f2 / 10, ("trapezoid not more accurate than Euler", e2, f2)


# --------------------------------------------------------------------------
# Mamba-2 (SSD): A is one number times the identity per head.  The pages
# ("State Space Models and the Post-Transformer Era", section "Mamba-2 and
# Structured State Space Duality") state that this scan is the same map as
# attention with a 1-semiseparable causal mask, computable either by the
# linear recurrence or by a quadratic matrix form.  Two pins: the quadratic
# form built with numpy matrix products, and the reduction to the S6 scan
# (pinned above) with A[d, n] = A[h] for every channel d of head h.


def _ssd_case(seed, softplus=True):
    rng = _rng(seed)
    bt, L, H, P, G, N = 2, 23, 4, 3, 2, 5
    return dict(
        x=rng.normal(size=(bt, L, H, P)), dt=rng.normal(size=(bt, L, H)),
        A=-rng.uniform(0.1, 1.5, size=H), B=rng.normal(size=(bt, L, G, N)),
        C=rng.normal(size=(bt, L, G, N)), D=rng.normal(size=H),
        z=rng.normal(size=(bt, L, H, P)), dt_bias=rng.normal(size=H) * 0.5,
        dt_softplus=softplus, h0=rng.normal(size=(bt, H, P, N)))


def pin_ssd_quadratic_form(lib):
    """y = (L o C B^T) (Delta x) plus the decayed initial state, per head:
    L[t, s] = exp(sum_{s<k<=t} Delta_k A), zero above the diagonal."""
    c = _ssd_case(31)
    bt, L, H, P = c["x"].shape
    G = c["B"].shape[2]
    want = np.zeros_like(c["x"])
    want_last = np.zeros_like(c["h0"])
    for b in range(bt):
        for h in range(H):
            g = h // (H // G)
            step = np.logaddexp(0.0, c["dt"][b, :, h] + c["dt_bias"][h])
            cum = np.cumsum(step * c["A"][h])
            mask = np.tril(np.exp(cum[:, None] - cum[None, :]))
            Bg, Cg, X = c["B"][b, :, g], c["C"][b, :, g], c["x"][b, :, h]
            M = (Cg @ Bg.T) * mask * step[None, :]
            yb = M @ X + np.exp(cum)[:, None] * (Cg @ c["h0"][b, h].T) + c["D"][h] * X
            want[b, :, h] = yb * c["z"][b, :, h] * scipy.special.expit(c["z"][b, :, h])
            w = np.exp(cum[-1] - cum) * step
            want_last[b, h] = np.exp(cum[-1]) * c["h0"][b, h] + (X * w[:, None]).T @ Bg
    got, got_last = oracle.ssd_scan(c["x"], c["dt"], c["A"], c["B"], c["C"], D=c["D"],
                                    z=c["z"], dt_bias=c["dt_bias"], h0=c["h0"],
                                    return_last_state=True, lib=lib)
    _close(got, want, 1e-9, 1e-12, "SSD quadratic form y")
    _close(got_last, want_last, 1e-9, 1e-12, "SSD quadratic form last state")


def pin_ssd_is_s6_with_scalar_A(lib):
    for softplus in (True, False):
        c = _ssd_case(32, softplus)
        if not softplus:
            c["dt"] = np.abs(c["dt"]) * 0.3 + 0.01
        bt, L, H, P = c["x"].shape
        G, N = c["B"].shape[2], c["B"].shape[3]
        got, got_last = oracle.ssd_scan(c["x"], c["dt"], c["A"], c["B"], c["C"], D=c["D"],
                                        z=c["z"], dt_bias=c["dt_bias"],
                                        dt_softplus=softplus, h0=c["h0"],
                                        return_last_state=True, lib=lib)
        for h in range(H):
            g = h // (H // G)
            y6, l6 = oracle.selective_scan(
                c["x"][:, :, h].transpose(0, 2, 1),
                np.repeat(c["dt"][:, None, :, h], P, axis=1),
                np.full((P, N), c["A"][h]),
                c["B"][:, :, g].transpose(0, 2, 1), c["C"][:, :, g].transpose(0, 2, 1),
                D=np.full(P, c["D"][h]), z=c["z"][:, :, h].transpose(0, 2, 1),
                delta_bias=np.full(P, c["dt_bias"][h]), delta_softplus=softplus,
                h0=c["h0"][:, h], return_last_state=True, lib=lib)
            _close(got[:, :, h], y6.transpose(0, 2, 1), 1e-12, 1e-14, "SSD vs S6 y")
            _close(got_last[:, h], l6, 1e-12, 1e-14, "SSD vs S6 last state")


ALL_PINS = [
    pin_combine_worked_example,
    pin_scan_worked_example,
    pin_state_update_worked_example,
    pin_state_update_special_cases,
    pin_combine_associative,
    pin_brute_force_unrolled,
    pin_lti_convolution,
    pin_n1_gate,
    pin_delta_limits,
    pin_special_cases,
    pin_softplus_silu,
    pin_resume,
    pin_packed_sequences,
    pin_backward_finite_differences,
    pin_trapezoid_no_decay,
    pin_trapezoid_second_order,
    pin_ssd_quadratic_form,
    pin_ssd_is_s6_with_scalar_A,
]
