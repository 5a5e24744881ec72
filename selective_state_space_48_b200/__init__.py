"""Python binding of the B200 selective-scan (S6) library.

Argument marshalling only: torch tensors supply device memory and the
current CUDA stream; every step of the computation runs in the CUDA kernels
of ``_lib/libsss48.so`` behind the C ABI declared in
``include/selective_scan.h``.  There is no CPU fallback: if the library is
missing or no CUDA device is present, the calls raise.

Functions mirror the C entry points:
  mamba_selective_scan_fwd  -> selective_scan_fwd(...)
  selective_state_update    -> selective_state_update(...)
  mss_scan_workspace_size   -> scan_workspace_size(...)
  mss_scan_status           -> scan_status(...)
  mamba2_ssd_fwd            -> ssd_fwd(...)         (include/ssd.h)
  mss_ssd_workspace_size    -> ssd_workspace_size(...)
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import builder as _build

LIB_PATH = _build.LIB_PATH

ABI_VERSION = 11  # MSS_ABI_VERSION of include/selective_scan.h

MSS_OK = 0
MSS_ERR_INVALID_ARG = 1
MSS_ERR_UNSUPPORTED = 2
MSS_ERR_CUDA = 3
MSS_ERR_TIMEOUT = 4
MSS_ERR_WORKSPACE = 5
MSS_F32 = 0
MSS_BF16 = 1
MSS_TESTFLAG_DROP_PUBLISH = 0x1
MSS_TESTFLAG_DEBUG_OOB = 0x2  # checked build only: one planted out-of-range y store

# every symbol include/selective_scan.h and include/ssd.h declare
EXPORTED_SYMBOLS = (
    "mss_scan_workspace_size",
    "mamba_selective_scan_fwd",
    "mss_scan_status",
    "mamba_selective_scan_fwd_noalloc",
    "mss_scan_noalloc_status",
    "selective_state_update",
    "mss_scan_bwd_workspace_size",
    "mamba_selective_scan_bwd",
    "mss_status_string",
    "mss_abi_version",
    "mss_ssd_workspace_size",
    "mamba2_ssd_fwd",
    "mss_ssd_status",
)


class ScanArgs(ctypes.Structure):
    """Mirror of ``mss_scan_args``."""
    _fields_ = [
        ("batch", ctypes.c_int64),
        ("dim", ctypes.c_int64),
        ("dstate", ctypes.c_int64),
        ("seqlen", ctypes.c_int64),
        ("in_dtype", ctypes.c_int),
        ("out_dtype", ctypes.c_int),
        ("u", ctypes.c_void_p),
        ("delta", ctypes.c_void_p),
        ("A", ctypes.c_void_p),
        ("B", ctypes.c_void_p),
        ("C", ctypes.c_void_p),
        ("D", ctypes.c_void_p),
        ("z", ctypes.c_void_p),
        ("delta_bias", ctypes.c_void_p),
        ("delta_softplus", ctypes.c_int),
        ("h0", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
        ("last_state", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("plan_splits", ctypes.c_int),
        ("plan_chunk_steps", ctypes.c_int),
        ("test_flags", ctypes.c_uint),
        ("spin_timeout_ns", ctypes.c_int64),
        ("stride_u", ctypes.c_int64 * 2),
        ("stride_delta", ctypes.c_int64 * 2),
        ("stride_z", ctypes.c_int64 * 2),
        ("stride_B", ctypes.c_int64 * 2),
        ("stride_C", ctypes.c_int64 * 2),
        ("stride_y", ctypes.c_int64 * 2),
        ("cu_seqlens", ctypes.c_void_p),
        ("num_seqs", ctypes.c_int64),
        ("trapezoid", ctypes.c_int),
        ("checkpoints", ctypes.c_void_p),
    ]


class UpdateArgs(ctypes.Structure):
    """Mirror of ``mss_update_args``."""
    _fields_ = [
        ("batch", ctypes.c_int64),
        ("dim", ctypes.c_int64),
        ("dstate", ctypes.c_int64),
        ("in_dtype", ctypes.c_int),
        ("out_dtype", ctypes.c_int),
        ("state", ctypes.c_void_p),
        ("x", ctypes.c_void_p),
        ("dt", ctypes.c_void_p),
        ("A", ctypes.c_void_p),
        ("B", ctypes.c_void_p),
        ("C", ctypes.c_void_p),
        ("D", ctypes.c_void_p),
        ("z", ctypes.c_void_p),
        ("dt_bias", ctypes.c_void_p),
        ("dt_softplus", ctypes.c_int),
        ("y", ctypes.c_void_p),
    ]


class ScanBwdArgs(ctypes.Structure):
    """Mirror of ``mss_scan_bwd_args``."""
    _fields_ = [
        ("batch", ctypes.c_int64),
        ("dim", ctypes.c_int64),
        ("dstate", ctypes.c_int64),
        ("seqlen", ctypes.c_int64),
        ("in_dtype", ctypes.c_int),
    ] + [(name, ctypes.c_void_p) for name in (
        "u", "delta", "A", "B", "C", "D", "z", "delta_bias")] + [
        ("delta_softplus", ctypes.c_int),
    ] + [(name, ctypes.c_void_p) for name in (
        "h0", "dy", "d_last", "du", "ddelta", "dA", "dB", "dC", "dD", "dz",
        "ddelta_bias", "dh0", "checkpoints", "workspace")] + [
        ("workspace_bytes", ctypes.c_size_t),
    ] + [("stride_" + name, ctypes.c_int64 * 2) for name in (
        "u", "delta", "z", "B", "C", "dy")] + [
        ("cu_seqlens", ctypes.c_void_p),
        ("num_seqs", ctypes.c_int64),
    ]


class SsdArgs(ctypes.Structure):
    """Mirror of ``mss_ssd_args``."""
    _fields_ = [(name, ctypes.c_int64) for name in (
        "batch", "seqlen", "nheads", "headdim", "ngroups", "dstate")] + [
        ("in_dtype", ctypes.c_int),
        ("out_dtype", ctypes.c_int),
    ] + [(name, ctypes.c_void_p) for name in (
        "x", "dt", "A", "B", "C", "D", "z", "dt_bias")] + [
        ("dt_softplus", ctypes.c_int),
    ] + [(name, ctypes.c_void_p) for name in ("h0", "y", "last_state")] + [
        ("spin_timeout_ns", ctypes.c_uint64),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
    ]


class MssError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)}")


_lib = None
_lock = threading.Lock()


def _bind(lib):
    P = ctypes.POINTER
    lib.mss_scan_workspace_size.argtypes = [P(ScanArgs), P(ctypes.c_size_t)]
    lib.mss_scan_workspace_size.restype = ctypes.c_int
    lib.mamba_selective_scan_fwd.argtypes = [P(ScanArgs), ctypes.c_void_p]
    lib.mamba_selective_scan_fwd.restype = ctypes.c_int
    lib.mss_scan_status.argtypes = [P(ScanArgs), ctypes.c_void_p]
    lib.mss_scan_status.restype = ctypes.c_int
    lib.mamba_selective_scan_fwd_noalloc.argtypes = [P(ScanArgs), ctypes.c_void_p]
    lib.mamba_selective_scan_fwd_noalloc.restype = ctypes.c_int
    lib.mss_scan_noalloc_status.argtypes = [P(ScanArgs), ctypes.c_void_p]
    lib.mss_scan_noalloc_status.restype = ctypes.c_int
    lib.selective_state_update.argtypes = [P(UpdateArgs), ctypes.c_void_p]
    lib.selective_state_update.restype = ctypes.c_int
    lib.mss_scan_bwd_workspace_size.argtypes = [P(ScanBwdArgs), P(ctypes.c_size_t)]
    lib.mss_scan_bwd_workspace_size.restype = ctypes.c_int
    lib.mamba_selective_scan_bwd.argtypes = [P(ScanBwdArgs), ctypes.c_void_p]
    lib.mamba_selective_scan_bwd.restype = ctypes.c_int
    lib.mss_status_string.argtypes = [ctypes.c_int]
    lib.mss_status_string.restype = ctypes.c_char_p
    lib.mss_ssd_workspace_size.argtypes = [P(SsdArgs), P(ctypes.c_size_t)]
    lib.mss_ssd_workspace_size.restype = ctypes.c_int
    lib.mamba2_ssd_fwd.argtypes = [P(SsdArgs), ctypes.c_void_p]
    lib.mamba2_ssd_fwd.restype = ctypes.c_int
    lib.mss_ssd_status.argtypes = [ctypes.c_void_p]
    lib.mss_ssd_status.restype = ctypes.c_int
    lib.mss_abi_version.argtypes = []
    lib.mss_abi_version.restype = ctypes.c_int
    return lib


def _open(path: str):
    if not os.path.exists(path):
        raise RuntimeError(
            f"CUDA library {path} is missing; build it with "
            "`python -m selective_state_space_48_b200.builder`")
    lib = _bind(ctypes.CDLL(path))
    if lib.mss_abi_version() != ABI_VERSION:
        raise RuntimeError(
            f"{path} has ABI version {lib.mss_abi_version()}, "
            f"this binding expects {ABI_VERSION}; rebuild it")
    return lib


def load_library():
    """Load libsss48.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = _open(LIB_PATH)
    return _lib


_debug_lib = None


def load_debug_library():
    """Load the checked build libsss48_debug.so (``builder --debug``): the
    same entry points with device-side bounds checks that report an access
    outside its tensor as MSS_ERR_INVALID_ARG through the status calls."""
    global _debug_lib
    with _lock:
        if _debug_lib is None:
            _debug_lib = _open(_build.DEBUG_LIB_PATH)
    return _debug_lib


def status_string(code: int) -> str:
    return load_library().mss_status_string(int(code)).decode()


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return MSS_F32
    if t == torch.bfloat16:
        return MSS_BF16
    raise TypeError(f"unsupported dtype {t}; use float32 or bfloat16")


def _ptr(t):
    return None if t is None else t.data_ptr()


def _check_cuda(name, t, dtype=None, shape=None, strided=False):
    """Type, dtype and shape checks; ``strided`` tensors may be views whose
    last (time) dimension is contiguous, all others must be contiguous."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if strided:
        if t.dim() != 3 or (t.shape[2] > 1 and t.stride(2) != 1):
            raise ValueError(f"{name} must be a 3-d view with a contiguous last dimension")
    elif not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_scan_args(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                   delta_softplus=True, h0=None, y=None, last_state=None,
                   workspace=None, plan_splits=0, test_flags=0,
                   spin_timeout_ns=0, cu_seqlens=None, trapezoid=False,
                   checkpoints=None) -> ScanArgs:
    batch, dim, L = u.shape
    N = A.shape[1]
    ind = u.dtype
    _check_cuda("u", u, ind, strided=True)
    _check_cuda("delta", delta, ind, (batch, dim, L), strided=True)
    _check_cuda("A", A, torch.float32, (dim, N))
    _check_cuda("B", B, ind, (batch, N, L), strided=True)
    _check_cuda("C", C, ind, (batch, N, L), strided=True)
    _check_cuda("D", D, torch.float32, (dim,))
    _check_cuda("z", z, ind, (batch, dim, L), strided=True)
    _check_cuda("delta_bias", delta_bias, torch.float32, (dim,))
    _check_cuda("h0", h0, torch.float32, (batch, dim, N))
    _check_cuda("last_state", last_state, torch.float32, (batch, dim, N))
    if y is not None:
        _check_cuda("y", y, None, (batch, dim, L), strided=True)
    a = ScanArgs()
    a.batch, a.dim, a.dstate, a.seqlen = batch, dim, N, L
    a.in_dtype = _dtype_code(ind)
    a.out_dtype = _dtype_code(y.dtype) if y is not None else MSS_F32
    a.u, a.delta, a.A, a.B, a.C = (_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C))
    a.D, a.z, a.delta_bias = _ptr(D), _ptr(z), _ptr(delta_bias)
    a.delta_softplus = 1 if delta_softplus else 0
    a.h0, a.y, a.last_state = _ptr(h0), _ptr(y), _ptr(last_state)
    if workspace is not None:
        a.workspace = workspace.data_ptr()
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    a.plan_splits = int(plan_splits)
    a.plan_chunk_steps = 0
    a.test_flags = int(test_flags)
    a.spin_timeout_ns = int(spin_timeout_ns)
    a.trapezoid = 1 if trapezoid else 0
    if checkpoints is not None:
        _check_cuda("checkpoints", checkpoints, torch.float32)
        a.checkpoints = checkpoints.data_ptr()
    if cu_seqlens is not None:
        _check_cuda("cu_seqlens", cu_seqlens, torch.int32)
        if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
            raise ValueError("cu_seqlens must hold num_seqs + 1 >= 2 offsets")
        a.cu_seqlens = cu_seqlens.data_ptr()
        a.num_seqs = cu_seqlens.numel() - 1
    for name, t in (("u", u), ("delta", delta), ("z", z), ("B", B), ("C", C), ("y", y)):
        if t is not None:
            getattr(a, "stride_" + name)[0] = t.stride(0)
            getattr(a, "stride_" + name)[1] = t.stride(1)
    return a


def scan_workspace_size(args: ScanArgs) -> int:
    n = ctypes.c_size_t(0)
    rc = load_library().mss_scan_workspace_size(ctypes.byref(args), ctypes.byref(n))
    if rc != MSS_OK:
        raise MssError(rc, "mss_scan_workspace_size")
    return int(n.value)


def alloc_workspace(nbytes: int, device) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    # torch allocations are 512-byte aligned, above the 256 the ABI needs
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def selective_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                       delta_softplus=True, h0=None, return_last_state=False,
                       out_dtype=torch.float32, y=None, last_state=None,
                       workspace=None, stream=None, plan_splits=0,
                       test_flags=0, spin_timeout_ns=0, check_status=False,
                       cu_seqlens=None, trapezoid=False, checkpoints=None):
    """Forward selective scan through ``mamba_selective_scan_fwd``.

    u, delta, z: (batch, dim, L); B, C: (batch, N, L) (float32 or bfloat16,
    all the same dtype); A: (dim, N), D, delta_bias: (dim,), h0:
    (batch, dim, N) float32.  u, delta, z, B, C and y may be views whose
    last dimension is contiguous.  ``cu_seqlens`` (int32 CUDA tensor of
    num_seqs + 1 offsets, 0 ... L) packs independent sequences into every
    row.  ``trapezoid`` selects the three-term trapezoidal update.
    ``checkpoints`` (from ``scan_checkpoints``) receives the states the
    backward pass starts from.  Returns
    y (batch, dim, L) in ``out_dtype`` (and the final state when
    ``return_last_state``).
    """
    batch, dim, L = u.shape
    N = A.shape[1]
    if y is None:
        y = torch.empty((batch, dim, L), dtype=out_dtype, device=u.device)
    if return_last_state and last_state is None:
        last_state = torch.empty((batch, dim, N), dtype=torch.float32,
                                 device=u.device)
    args = make_scan_args(u, delta, A, B, C, D, z, delta_bias, delta_softplus,
                          h0, y, last_state, None, plan_splits, test_flags,
                          spin_timeout_ns, cu_seqlens, trapezoid, checkpoints)
    if workspace is None:
        workspace = alloc_workspace(scan_workspace_size(args), u.device)
    if workspace is not None:
        args.workspace = workspace.data_ptr()
        args.workspace_bytes = workspace.numel() * workspace.element_size()
    lib = load_library()
    rc = lib.mamba_selective_scan_fwd(ctypes.byref(args), _stream_handle(stream))
    if rc != MSS_OK:
        raise MssError(rc, "mamba_selective_scan_fwd")
    if check_status:
        rc = lib.mss_scan_status(ctypes.byref(args), _stream_handle(stream))
        if rc != MSS_OK:
            raise MssError(rc, "mss_scan_status")
    # keep the workspace alive until the stream has used it
    if workspace is not None:
        workspace.record_stream(stream or torch.cuda.current_stream())
    return (y, last_state) if return_last_state else y


def scan_status(args: ScanArgs, stream=None) -> int:
    """Raw status code of the last scan that used ``args.workspace``."""
    return load_library().mss_scan_status(ctypes.byref(args), _stream_handle(stream))


def selective_state_update(state, x, dt, A, B, C, D=None, z=None, dt_bias=None,
                           dt_softplus=True, out_dtype=torch.float32, y=None,
                           stream=None):
    """One decode step through ``selective_state_update``; ``state``
    (batch, dim, N) float32 is updated in place.  x, dt, z: (batch, dim);
    B, C: (batch, N).  Returns y (batch, dim)."""
    batch, dim, N = state.shape
    ind = x.dtype
    _check_cuda("state", state, torch.float32)
    _check_cuda("x", x, ind, (batch, dim))
    _check_cuda("dt", dt, ind, (batch, dim))
    _check_cuda("A", A, torch.float32, (dim, N))
    _check_cuda("B", B, ind, (batch, N))
    _check_cuda("C", C, ind, (batch, N))
    _check_cuda("D", D, torch.float32, (dim,))
    _check_cuda("z", z, ind, (batch, dim))
    _check_cuda("dt_bias", dt_bias, torch.float32, (dim,))
    if y is None:
        y = torch.empty((batch, dim), dtype=out_dtype, device=state.device)
    _check_cuda("y", y, None, (batch, dim))
    a = UpdateArgs()
    a.batch, a.dim, a.dstate = batch, dim, N
    a.in_dtype, a.out_dtype = _dtype_code(ind), _dtype_code(y.dtype)
    a.state, a.x, a.dt = _ptr(state), _ptr(x), _ptr(dt)
    a.A, a.B, a.C, a.D, a.z = _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z)
    a.dt_bias = _ptr(dt_bias)
    a.dt_softplus = 1 if dt_softplus else 0
    a.y = _ptr(y)
    rc = load_library().selective_state_update(ctypes.byref(a), _stream_handle(stream))
    if rc != MSS_OK:
        raise MssError(rc, "selective_state_update")
    return y


def make_ssd_args(x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True,
                  h0=None, y=None, last_state=None, spin_timeout_ns=0) -> SsdArgs:
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    ind = x.dtype
    _check_cuda("x", x, ind)
    _check_cuda("dt", dt, ind, (batch, L, H))
    _check_cuda("A", A, torch.float32, (H,))
    _check_cuda("B", B, ind, (batch, L, G, N))
    _check_cuda("C", C, ind, (batch, L, G, N))
    _check_cuda("D", D, torch.float32, (H,))
    _check_cuda("z", z, ind, (batch, L, H, P))
    _check_cuda("dt_bias", dt_bias, torch.float32, (H,))
    _check_cuda("h0", h0, torch.float32, (batch, H, P, N))
    _check_cuda("last_state", last_state, torch.float32, (batch, H, P, N))
    if y is not None:
        _check_cuda("y", y, None, (batch, L, H, P))
    a = SsdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.ngroups, a.dstate = batch, L, H, P, G, N
    a.in_dtype = _dtype_code(ind)
    a.out_dtype = _dtype_code(y.dtype) if y is not None else MSS_F32
    a.x, a.dt, a.A, a.B, a.C = _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C)
    a.D, a.z, a.dt_bias = _ptr(D), _ptr(z), _ptr(dt_bias)
    a.dt_softplus = 1 if dt_softplus else 0
    a.h0, a.y, a.last_state = _ptr(h0), _ptr(y), _ptr(last_state)
    a.spin_timeout_ns = int(spin_timeout_ns)
    return a


def ssd_workspace_size(args: SsdArgs) -> int:
    """``mss_ssd_workspace_size``: bytes that let the SSD scan cut the last
    wave's sequences in two on the current device (0: nothing to cut)."""
    n = ctypes.c_size_t(0)
    rc = load_library().mss_ssd_workspace_size(ctypes.byref(args), ctypes.byref(n))
    if rc != MSS_OK:
        raise MssError(rc, "mss_ssd_workspace_size")
    return int(n.value)


def ssd_fwd(x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True, h0=None,
            return_last_state=False, out_dtype=torch.float32, y=None, last_state=None,
            stream=None, check_status=False, workspace=None):
    """Mamba-2 (SSD) chunked scan through ``mamba2_ssd_fwd``.

    x, z: (batch, L, nheads, headdim); dt: (batch, L, nheads); B, C:
    (batch, L, ngroups, dstate), all bfloat16; A, D, dt_bias: (nheads,)
    float32; h0: (batch, nheads, headdim, dstate) float32.  Returns y
    (batch, L, nheads, headdim) in ``out_dtype`` (and the final state when
    ``return_last_state``).  ``workspace``: None allocates what
    ``ssd_workspace_size`` asks for; False runs every sequence whole; a
    uint8 CUDA tensor is used as given.
    """
    batch, L, H, P = x.shape
    N = B.shape[3]
    if y is None:
        y = torch.empty((batch, L, H, P), dtype=out_dtype, device=x.device)
    if return_last_state and last_state is None:
        last_state = torch.empty((batch, H, P, N), dtype=torch.float32, device=x.device)
    args = make_ssd_args(x, dt, A, B, C, D, z, dt_bias, dt_softplus, h0, y, last_state)
    if workspace is None:
        workspace = alloc_workspace(ssd_workspace_size(args), x.device)
    if workspace is not None and workspace is not False:
        args.workspace = workspace.data_ptr()
        args.workspace_bytes = workspace.numel() * workspace.element_size()
    lib = load_library()
    rc = lib.mamba2_ssd_fwd(ctypes.byref(args), _stream_handle(stream))
    if rc != MSS_OK:
        raise MssError(rc, "mamba2_ssd_fwd")
    # keep the workspace alive until the stream has used it
    if workspace is not None and workspace is not False:
        workspace.record_stream(stream or torch.cuda.current_stream())
    if check_status:
        rc = lib.mss_ssd_status(_stream_handle(stream))
        if rc != MSS_OK:
            raise MssError(rc, "mss_ssd_status")
    return (y, last_state) if return_last_state else y


def build(force: bool = False) -> str:
    return _build.build(force=force)


__all__ = [
    "selective_scan_fwd", "selective_state_update", "scan_workspace_size",
    "scan_status", "make_scan_args", "load_library", "status_string",
    "MssError", "ScanArgs", "UpdateArgs", "EXPORTED_SYMBOLS", "build",
    "ssd_fwd", "make_ssd_args", "SsdArgs", "ssd_workspace_size",
]


def selective_scan_bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None,
                       delta_softplus=True, h0=None, d_last=None, stream=None,
                       workspace=None, checkpoints=None, cu_seqlens=None):
    """Gradients of sum(dy * y) + sum(d_last * last_state) for the forward
    scan on the same inputs (and the same ``cu_seqlens`` packing), through
    ``mamba_selective_scan_bwd``.

    Inputs as for ``selective_scan_fwd`` (u, delta, z, B, C and dy may be
    3-d views with a contiguous last dimension); dy (batch, dim, L) and
    d_last (batch, dim, N) float32.  ``checkpoints`` written by the forward
    scan of the same inputs let the backward skip its forward sweep.
    ``workspace``: None allocates what ``mss_scan_bwd_workspace_size`` asks
    for (the checkpoints and the cut schedule's area); False passes none
    (valid with ``checkpoints``; every tile then runs whole); a uint8 CUDA
    tensor is used as given.  Returns a dict of float32 tensors du, ddelta,
    dA, dB, dC, dD, dz, ddelta_bias, dh0 (None for absent inputs).
    """
    batch, dim, L = u.shape
    N = A.shape[1]
    ind = u.dtype
    rows = ("u", "delta", "B", "C", "z", "dy")  # may be strided views
    for name, t, dt, shape in (
            ("u", u, ind, None), ("delta", delta, ind, (batch, dim, L)),
            ("A", A, torch.float32, (dim, N)), ("B", B, ind, (batch, N, L)),
            ("C", C, ind, (batch, N, L)), ("D", D, torch.float32, (dim,)),
            ("z", z, ind, (batch, dim, L)),
            ("delta_bias", delta_bias, torch.float32, (dim,)),
            ("h0", h0, torch.float32, (batch, dim, N)),
            ("dy", dy, torch.float32, (batch, dim, L)),
            ("d_last", d_last, torch.float32, (batch, dim, N))):
        _check_cuda(name, t, dt, shape, strided=name in rows)
    dev = u.device
    f32 = dict(dtype=torch.float32, device=dev)
    g = {
        "du": torch.empty((batch, dim, L), **f32),
        "ddelta": torch.empty((batch, dim, L), **f32),
        "dA": torch.empty((dim, N), **f32),
        "dB": torch.empty((batch, N, L), **f32),
        "dC": torch.empty((batch, N, L), **f32),
        "dD": torch.empty((dim,), **f32) if D is not None else None,
        "dz": torch.empty((batch, dim, L), **f32) if z is not None else None,
        "ddelta_bias": torch.empty((dim,), **f32) if delta_bias is not None else None,
        "dh0": torch.empty((batch, dim, N), **f32),
    }
    a = ScanBwdArgs()
    a.batch, a.dim, a.dstate, a.seqlen = batch, dim, N, L
    a.in_dtype = _dtype_code(ind)
    a.u, a.delta, a.A, a.B, a.C = _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C)
    a.D, a.z, a.delta_bias = _ptr(D), _ptr(z), _ptr(delta_bias)
    a.delta_softplus = 1 if delta_softplus else 0
    a.h0, a.dy, a.d_last = _ptr(h0), _ptr(dy), _ptr(d_last)
    a.checkpoints = _ptr(checkpoints)
    for k, v in g.items():
        setattr(a, k, _ptr(v))
    for name, t in (("u", u), ("delta", delta), ("z", z), ("B", B), ("C", C), ("dy", dy)):
        if t is not None:
            getattr(a, "stride_" + name)[0] = t.stride(0)
            getattr(a, "stride_" + name)[1] = t.stride(1)
    if cu_seqlens is not None:
        _check_cuda("cu_seqlens", cu_seqlens, torch.int32)
        if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
            raise ValueError("cu_seqlens must hold num_seqs + 1 >= 2 offsets")
        a.cu_seqlens = cu_seqlens.data_ptr()
        a.num_seqs = cu_seqlens.numel() - 1
    lib = load_library()
    n = ctypes.c_size_t(0)
    rc = lib.mss_scan_bwd_workspace_size(ctypes.byref(a), ctypes.byref(n))
    if rc != MSS_OK:
        raise MssError(rc, "mss_scan_bwd_workspace_size")
    if workspace is None:
        # the checkpoints (without given ones) and the cut schedule's area
        workspace = alloc_workspace(int(n.value), dev)
    if workspace is False:  # no workspace (valid with checkpoints): no cut
        workspace = None
    if workspace is not None:
        a.workspace = workspace.data_ptr()
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    rc = lib.mamba_selective_scan_bwd(ctypes.byref(a), _stream_handle(stream))
    if rc != MSS_OK:
        raise MssError(rc, "mamba_selective_scan_bwd")
    if workspace is not None:
        workspace.record_stream(stream or torch.cuda.current_stream())
    return g


def scan_checkpoints(batch, dim, dstate, seqlen, device):
    """A buffer for the forward scan's checkpoints (float32, the checkpoint
    part of what ``mss_scan_bwd_workspace_size`` reports)."""
    groups = (dstate + 3) // 4
    groups = 1 if groups <= 1 else (2 if groups == 2 else 4)
    tiles = batch * ((dim + 31) // 32)
    nblk = (seqlen + 15) // 16
    # two arrays: the states at every block's start and entering its step 8
    return torch.empty(2 * tiles * nblk * 4 * groups * 32, dtype=torch.float32,
                       device=device)


class _SelectiveScanFn(torch.autograd.Function):
    """Autograd wrapper: forward through mamba_selective_scan_fwd (writing
    the backward's state checkpoints), backward through
    mamba_selective_scan_bwd starting from them."""

    @staticmethod
    def forward(ctx, u, delta, A, B, C, D, z, delta_bias, delta_softplus, h0, cu_seqlens):
        batch, dim, L = u.shape
        # packed sequences: no forward checkpoints, the backward sweeps itself
        ck = (scan_checkpoints(batch, dim, A.shape[1], L, u.device)
              if cu_seqlens is None else None)
        y = selective_scan_fwd(u, delta, A, B, C, D=D, z=z, delta_bias=delta_bias,
                               delta_softplus=delta_softplus, h0=h0, checkpoints=ck,
                               cu_seqlens=cu_seqlens)
        ctx.delta_softplus = delta_softplus
        ctx.save_for_backward(u, delta, A, B, C, D, z, delta_bias, h0, ck, cu_seqlens)
        return y

    @staticmethod
    def backward(ctx, dy):
        u, delta, A, B, C, D, z, delta_bias, h0, ck, cu = ctx.saved_tensors
        g = selective_scan_bwd(u, delta, A, B, C, _rows_view(dy.float()), D=D, z=z,
                               delta_bias=delta_bias, delta_softplus=ctx.delta_softplus,
                               h0=h0, checkpoints=ck, cu_seqlens=cu)
        cast = lambda t, like: None if t is None else t.to(like.dtype)
        return (cast(g["du"], u), cast(g["ddelta"], delta), g["dA"], cast(g["dB"], B),
                cast(g["dC"], C), g["dD"], cast(g["dz"], z) if z is not None else None,
                g["ddelta_bias"], None, g["dh0"] if h0 is not None else None, None)


def _rows_view(t):
    """t itself when its last (time) dimension is contiguous, else a copy."""
    return t if t.dim() == 3 and (t.shape[2] <= 1 or t.stride(2) == 1) else t.contiguous()


def selective_scan_fn(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                      delta_softplus=True, h0=None, cu_seqlens=None):
    """Differentiable selective scan: y (batch, dim, L) float32, with
    gradients for every tensor input through the CUDA backward pass.
    Inputs as for ``selective_scan_fwd``: u, delta, B, C and z may be views
    with a contiguous time dimension (the halves of an input projection,
    say), which both passes read in place; ``cu_seqlens`` packs independent
    sequences as for ``selective_scan_fwd``.  Gradients come back packed, in
    the inputs' dtypes (computed in float32)."""
    return _SelectiveScanFn.apply(_rows_view(u), _rows_view(delta), A, _rows_view(B),
                                  _rows_view(C), D, None if z is None else _rows_view(z),
                                  delta_bias, delta_softplus, h0, cu_seqlens)
