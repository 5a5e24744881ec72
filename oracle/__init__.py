"""fp64 CPU oracle of the selective scan (S6) -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never loads it, and it imports nothing from them.

The arithmetic lives in ``oracle.c`` (plain C, double precision, OpenMP over
independent channels).  This module only compiles it with gcc and passes
numpy float64 arrays to it.  Which page and section each step follows is
stated in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_HDR = os.path.join(_HERE, "oracle.h")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

_lib = None
_lock = threading.Lock()

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.c_int64


def build(force: bool = False, src: str | None = None, out: str | None = None,
          openmp: bool = True) -> str:
    """Compile the oracle into a shared library with gcc; returns its path.

    ``src``/``out`` let a test compile a modified copy of the source.
    """
    src = src or _SRC
    out = out or _LIB_PATH
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= max(os.path.getmtime(src),
                                             os.path.getmtime(_HDR))):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-I", _HERE,
           "-fno-fast-math", "-ffp-contract=off"]
    if openmp:
        cmd.append("-fopenmp")
    tmp = out + f".tmp{os.getpid()}"
    cmd += [src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    os.replace(tmp, out)
    return out


def _bind(lib):
    lib.oracle_combine_f64.argtypes = [ctypes.c_double] * 4 + [_D, _D]
    lib.oracle_combine_f64.restype = None
    lib.oracle_softplus_f64.argtypes = [ctypes.c_double]
    lib.oracle_softplus_f64.restype = ctypes.c_double
    lib.oracle_silu_f64.argtypes = [ctypes.c_double]
    lib.oracle_silu_f64.restype = ctypes.c_double
    lib.oracle_selective_scan_f64.argtypes = (
        [_I64] * 4 + [_D] * 8 + [ctypes.c_int, _D, _D, _D,
                                 ctypes.POINTER(ctypes.c_int32), _I64, ctypes.c_int])
    lib.oracle_selective_scan_f64.restype = ctypes.c_int
    lib.oracle_selective_state_update_f64.argtypes = (
        [_I64] * 3 + [_D] * 9 + [ctypes.c_int, _D])
    lib.oracle_selective_state_update_f64.restype = ctypes.c_int
    lib.oracle_selective_scan_bwd_f64.argtypes = (
        [_I64] * 4 + [_D] * 8 + [ctypes.c_int] + [_D] * 12 +
        [ctypes.POINTER(ctypes.c_int32), _I64])
    lib.oracle_selective_scan_bwd_f64.restype = ctypes.c_int
    lib.oracle_ssd_scan_f64.argtypes = (
        [_I64] * 6 + [_D] * 8 + [ctypes.c_int, _D, _D, _D])
    lib.oracle_ssd_scan_f64.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
    lib.oracle_set_num_threads.restype = None
    return lib


def load(path: str | None = None):
    """Load (building if needed) the oracle library.  ``path`` loads another
    compiled copy (used by the planted-mistake tests)."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(_D)


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def combine(a1, b1, a2, b2, lib=None):
    """(a1, b1) then (a2, b2) -> (a1 a2, a2 b1 + b2)."""
    lib = lib or load()
    a = ctypes.c_double()
    b = ctypes.c_double()
    lib.oracle_combine_f64(a1, b1, a2, b2, ctypes.byref(a), ctypes.byref(b))
    return a.value, b.value


def softplus(x, lib=None):
    lib = lib or load()
    return lib.oracle_softplus_f64(float(x))


def silu(z, lib=None):
    lib = lib or load()
    return lib.oracle_silu_f64(float(z))


def selective_scan(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                   delta_softplus=True, h0=None, return_last_state=False,
                   lib=None, cu_seqlens=None, trapezoid=False):
    """Sequential fp64 selective scan.

    u, delta, z: (batch, dim, L); B, C: (batch, N, L); A: (dim, N);
    D, delta_bias: (dim,); h0: (batch, dim, N).  Returns y (batch, dim, L)
    float64, and the final state when ``return_last_state``.  cu_seqlens
    (num_seqs + 1 offsets, 0 ... L) packs independent sequences into every
    row: the state restarts from zero at each interior offset.
    ``trapezoid`` selects the three-term trapezoidal update.
    """
    lib = lib or load()
    u = _f64(u)
    delta = _f64(delta)
    A = _f64(A)
    B = _f64(B)
    C = _f64(C)
    D = _f64(D)
    z = _f64(z)
    delta_bias = _f64(delta_bias)
    h0 = _f64(h0)
    batch, dim, L = u.shape
    N = A.shape[1]
    assert delta.shape == u.shape and A.shape == (dim, N)
    assert B.shape == (batch, N, L) and C.shape == (batch, N, L)
    y = np.empty((batch, dim, L), dtype=np.float64)
    last = (np.empty((batch, dim, N), dtype=np.float64)
            if return_last_state else None)
    cu, nseq = None, 0
    if cu_seqlens is not None:
        cu_arr = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        nseq = len(cu_arr) - 1
        cu = cu_arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    rc = lib.oracle_selective_scan_f64(
        batch, dim, N, L, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
        _ptr(D), _ptr(z), _ptr(delta_bias), int(bool(delta_softplus)),
        _ptr(h0), _ptr(y), _ptr(last), cu, nseq, int(bool(trapezoid)))
    if rc != 0:
        raise ValueError("oracle_selective_scan_f64 rejected the sizes")
    return (y, last) if return_last_state else y


def selective_state_update(state, x, dt, A, B, C, D=None, z=None,
                           dt_bias=None, dt_softplus=True, lib=None):
    """One fp64 decode step.  Returns (new_state, y); ``state`` is not
    modified (a copy is updated)."""
    lib = lib or load()
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    x = _f64(x)
    dt = _f64(dt)
    A = _f64(A)
    B = _f64(B)
    C = _f64(C)
    D = _f64(D)
    z = _f64(z)
    dt_bias = _f64(dt_bias)
    batch, dim, N = st.shape
    y = np.empty((batch, dim), dtype=np.float64)
    rc = lib.oracle_selective_state_update_f64(
        batch, dim, N, _ptr(st), _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
        _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias), int(bool(dt_softplus)),
        _ptr(y))
    if rc != 0:
        raise ValueError("oracle_selective_state_update_f64 rejected sizes")
    return st, y


def num_threads(lib=None) -> int:
    lib = lib or load()
    return int(lib.oracle_num_threads())


def set_num_threads(n: int, lib=None) -> None:
    """Threads of later oracle calls (e.g. 1 to time it on one core)."""
    lib = lib or load()
    lib.oracle_set_num_threads(int(n))


def selective_scan_bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None,
                       delta_softplus=True, h0=None, d_last=None, lib=None,
                       cu_seqlens=None):
    """fp64 gradient of ``selective_scan`` (with the same ``cu_seqlens``
    packing) for the loss sum(dy * y) + sum(d_last * last_state).  Returns a
    dict with du, ddelta, dA, dB, dC, dD, dz, ddelta_bias, dh0 (None where
    the input is absent)."""
    lib = lib or load()
    u, delta, A, B, C, dy = (_f64(x) for x in (u, delta, A, B, C, dy))
    D, z, delta_bias, h0, d_last = (_f64(x) for x in (D, z, delta_bias, h0, d_last))
    batch, dim, L = u.shape
    N = A.shape[1]
    out = {
        "du": np.empty((batch, dim, L)), "ddelta": np.empty((batch, dim, L)),
        "dA": np.empty((dim, N)), "dB": np.empty((batch, N, L)),
        "dC": np.empty((batch, N, L)),
        "dD": np.empty(dim) if D is not None else None,
        "dz": np.empty((batch, dim, L)) if z is not None else None,
        "ddelta_bias": np.empty(dim) if delta_bias is not None else None,
        "dh0": np.empty((batch, dim, N)),
    }
    cu, nseq = None, 0
    if cu_seqlens is not None:
        cu_arr = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        nseq = len(cu_arr) - 1
        cu = cu_arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    rc = lib.oracle_selective_scan_bwd_f64(
        batch, dim, N, L, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
        _ptr(D), _ptr(z), _ptr(delta_bias), int(bool(delta_softplus)),
        _ptr(h0), _ptr(dy), _ptr(d_last), _ptr(out["du"]), _ptr(out["ddelta"]),
        _ptr(out["dA"]), _ptr(out["dB"]), _ptr(out["dC"]), _ptr(out["dD"]),
        _ptr(out["dz"]), _ptr(out["ddelta_bias"]), _ptr(out["dh0"]), cu, nseq)
    if rc != 0:
        raise ValueError("oracle_selective_scan_bwd_f64 rejected the sizes")
    return out


def ssd_scan(x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True,
             h0=None, return_last_state=False, lib=None):
    """Sequential fp64 Mamba-2 (SSD) scan: A is one scalar per head.

    x, z: (batch, L, nheads, headdim); dt: (batch, L, nheads);
    A, D, dt_bias: (nheads,); B, C: (batch, L, ngroups, dstate);
    h0: (batch, nheads, headdim, dstate).  Returns y (batch, L, nheads,
    headdim) float64, and the final state when ``return_last_state``.
    """
    lib = lib or load()
    x, dt, A, B, C = (_f64(a) for a in (x, dt, A, B, C))
    D, z, dt_bias, h0 = (_f64(a) for a in (D, z, dt_bias, h0))
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert dt.shape == (batch, L, H) and A.shape == (H,)
    assert B.shape == (batch, L, G, N) and C.shape == B.shape
    y = np.empty((batch, L, H, P), dtype=np.float64)
    last = np.empty((batch, H, P, N), dtype=np.float64) if return_last_state else None
    rc = lib.oracle_ssd_scan_f64(
        batch, L, H, P, G, N, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
        _ptr(D), _ptr(z), _ptr(dt_bias), int(bool(dt_softplus)), _ptr(h0),
        _ptr(y), _ptr(last))
    if rc != 0:
        raise ValueError("oracle_ssd_scan_f64 rejected the sizes")
    return (y, last) if return_last_state else y
