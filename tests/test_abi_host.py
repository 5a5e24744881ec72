"""Host-side checks of the C ABI (no GPU needed, no compute launched).

* the library builds and loads, and exports every function the header
  declares;
* the ctypes mirrors of the argument structs have the C layout;
* argument checks reject bad calls before touching the device.
"""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

import selective_state_space_48_b200 as sss
from selective_state_space_48_b200 import builder as sbuild

HEADER_DIR = sbuild.INCLUDE


@pytest.fixture(scope="module")
def lib():
    sbuild.build()
    return sss.load_library()


def declared_functions():
    names = []
    for fn in os.listdir(HEADER_DIR):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(HEADER_DIR, fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b([A-Za-z_]\w*)\s*\([^;{]*\)\s*;",
                             text, flags=re.M):
            names.append(m.group(1))
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for sym in sss.EXPORTED_SYMBOLS:
        assert sym in names
    assert set(names) == set(sss.EXPORTED_SYMBOLS), names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", sbuild.LIB_PATH],
                         capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for sym in declared_functions():
        assert sym in exported, sym
        assert getattr(lib, sym) is not None


def test_checked_build_exports_the_same_symbols():
    """The checked build (MSS_DEBUG=1: device-side bounds checks) is the same
    library: it loads, has this ABI version and exports every declared entry
    point.  Built here if build() has not built it yet (nvcc, no GPU)."""
    path = sbuild.build(debug=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path],
                         capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for sym in declared_functions():
        assert sym in exported, sym
    dbg = sss.load_debug_library()
    assert dbg.mss_abi_version() == sss.ABI_VERSION


def test_abi_version_and_status_strings(lib):
    assert lib.mss_abi_version() == sss.ABI_VERSION == 11
    for code, name in [(0, "MSS_OK"), (1, "MSS_ERR_INVALID_ARG"),
                       (2, "MSS_ERR_UNSUPPORTED"), (3, "MSS_ERR_CUDA"),
                       (4, "MSS_ERR_TIMEOUT"), (5, "MSS_ERR_WORKSPACE")]:
        assert sss.status_string(code) == name


def test_struct_layout_matches_c():
    """Compile a C program that prints sizeof/offsetof of the structs."""
    fields_scan = [f[0] for f in sss.ScanArgs._fields_]
    fields_upd = [f[0] for f in sss.UpdateArgs._fields_]
    fields_bwd = [f[0] for f in sss.ScanBwdArgs._fields_]
    fields_ssd = [f[0] for f in sss.SsdArgs._fields_]
    src = ['#include <stdio.h>', '#include <stddef.h>', '#include "ssd.h"',
           'int main(void) {',
           'printf("%zu\\n", sizeof(mss_scan_args));']
    src += [f'printf("%zu\\n", offsetof(mss_scan_args, {f}));' for f in fields_scan]
    src += ['printf("%zu\\n", sizeof(mss_update_args));']
    src += [f'printf("%zu\\n", offsetof(mss_update_args, {f}));' for f in fields_upd]
    src += ['printf("%zu\\n", sizeof(mss_scan_bwd_args));']
    src += [f'printf("%zu\\n", offsetof(mss_scan_bwd_args, {f}));' for f in fields_bwd]
    src += ['printf("%zu\\n", sizeof(mss_ssd_args));']
    src += [f'printf("%zu\\n", offsetof(mss_ssd_args, {f}));' for f in fields_ssd]
    src += ['return 0; }']
    with tempfile.TemporaryDirectory() as tmp:
        c = os.path.join(tmp, "layout.c")
        exe = os.path.join(tmp, "layout")
        open(c, "w").write("\n".join(src))
        subprocess.run(["gcc", "-I", HEADER_DIR, c, "-o", exe], check=True)
        vals = [int(v) for v in subprocess.run([exe], capture_output=True, text=True,
                                               check=True).stdout.split()]
    want = [ctypes.sizeof(sss.ScanArgs)] + [getattr(sss.ScanArgs, f).offset for f in fields_scan]
    want += [ctypes.sizeof(sss.UpdateArgs)] + [getattr(sss.UpdateArgs, f).offset for f in fields_upd]
    want += [ctypes.sizeof(sss.ScanBwdArgs)] + [getattr(sss.ScanBwdArgs, f).offset for f in fields_bwd]
    want += [ctypes.sizeof(sss.SsdArgs)] + [getattr(sss.SsdArgs, f).offset for f in fields_ssd]
    assert vals == want


def _args(**kw):
    a = sss.ScanArgs()
    a.batch, a.dim, a.dstate, a.seqlen = 2, 40, 16, 4096
    a.in_dtype, a.out_dtype = sss.MSS_BF16, sss.MSS_F32
    fake = 0x10000
    a.u = a.delta = a.A = a.B = a.C = a.y = fake
    a.plan_splits = 4
    for k, v in kw.items():
        if k.startswith("stride_"):
            getattr(a, k)[0], getattr(a, k)[1] = v
        else:
            setattr(a, k, v)
    return a


def _ws(lib, a):
    n = ctypes.c_size_t(123)
    rc = lib.mss_scan_workspace_size(ctypes.byref(a), ctypes.byref(n))
    return rc, n.value


def test_workspace_size_follows_plan(lib):
    rc, n = _ws(lib, _args(plan_splits=1))
    assert rc == sss.MSS_OK and n == 0
    rc, n4 = _ws(lib, _args(plan_splits=4))
    assert rc == sss.MSS_OK and n4 > 0
    rc, n8 = _ws(lib, _args(plan_splits=8))
    assert rc == sss.MSS_OK and n8 > n4
    # 2 batch rows x 2 channel tiles x 8 chunks, each with (P, e) and the
    # true end state for 32 channels x 16 states (plus the running sums of
    # Delta at the chunk's segment starts)
    items = 2 * 2 * 8
    assert n8 >= items * 32 * 16 * 3 * 4


@pytest.mark.parametrize("kw,code", [
    (dict(batch=0), sss.MSS_ERR_INVALID_ARG),
    (dict(dim=0), sss.MSS_ERR_INVALID_ARG),
    (dict(seqlen=0), sss.MSS_ERR_INVALID_ARG),
    (dict(dstate=0), sss.MSS_ERR_INVALID_ARG),
    (dict(dstate=17), sss.MSS_ERR_UNSUPPORTED),
    (dict(in_dtype=7), sss.MSS_ERR_INVALID_ARG),
    (dict(out_dtype=-1), sss.MSS_ERR_INVALID_ARG),
    (dict(u=0), sss.MSS_ERR_INVALID_ARG),
    (dict(y=0), sss.MSS_ERR_INVALID_ARG),
    (dict(A=0x10002), sss.MSS_ERR_INVALID_ARG),      # fp32 A misaligned
    (dict(u=0x10001), sss.MSS_ERR_INVALID_ARG),      # bf16 u misaligned
    (dict(plan_splits=-1), sss.MSS_ERR_INVALID_ARG),
    (dict(plan_chunk_steps=64), sss.MSS_ERR_INVALID_ARG),
    (dict(spin_timeout_ns=-5), sss.MSS_ERR_INVALID_ARG),
    (dict(stride_u=(-1, 4096)), sss.MSS_ERR_INVALID_ARG),       # negative stride
    (dict(stride_B=(0, -4096)), sss.MSS_ERR_INVALID_ARG),
    (dict(stride_y=(40 * 4096, 4095)), sss.MSS_ERR_INVALID_ARG),  # y rows overlap
    (dict(stride_y=(39 * 4096, 4096)), sss.MSS_ERR_INVALID_ARG),  # y batches overlap
    (dict(stride_y=(0, 4096)), sss.MSS_ERR_INVALID_ARG),          # y batches alias
    (dict(stride_z=(1 << 50, 4096)), sss.MSS_ERR_INVALID_ARG),    # absurd
    (dict(num_seqs=3), sss.MSS_ERR_INVALID_ARG),                  # offsets missing
    (dict(cu_seqlens=0x10000, num_seqs=0), sss.MSS_ERR_INVALID_ARG),
    (dict(cu_seqlens=0x10002, num_seqs=2), sss.MSS_ERR_INVALID_ARG),  # misaligned
    (dict(trapezoid=2), sss.MSS_ERR_INVALID_ARG),
    (dict(trapezoid=1, cu_seqlens=0x10000, num_seqs=2), sss.MSS_ERR_UNSUPPORTED),
    (dict(checkpoints=0x10000, trapezoid=1), sss.MSS_ERR_UNSUPPORTED),
    (dict(checkpoints=0x10002), sss.MSS_ERR_INVALID_ARG),           # misaligned
    (dict(checkpoints=0x10000, plan_splits=3), sss.MSS_ERR_INVALID_ARG),
])
def test_bad_arguments_are_rejected_before_launch(lib, kw, code):
    a = _args(**kw)
    rc, _ = _ws(lib, a)
    assert rc == code
    # the forward call applies the same checks and launches nothing
    assert lib.mamba_selective_scan_fwd(ctypes.byref(a), None) == code


@pytest.mark.parametrize("kw", [
    dict(stride_u=(80 * 4096, 4096)),          # u: half of a (2, 80, L) projection
    dict(stride_z=(80 * 4096, 4096)),
    dict(stride_B=(0, 4096)),                  # one B shared by the batch rows
    dict(stride_C=(16 * 4096, 4096 + 8)),      # padded rows
    dict(stride_y=(41 * 4100, 4100)),          # y inside a larger buffer
    dict(stride_delta=(0, 0)),                 # packed
    dict(cu_seqlens=0x10000, num_seqs=5),      # packed sequences
    dict(trapezoid=1),                         # three-term update
    dict(checkpoints=0x10000),                 # states for the backward
])
def test_valid_strides_are_accepted(lib, kw):
    rc, n = _ws(lib, _args(plan_splits=1, **kw))
    assert rc == sss.MSS_OK and n == 0


def test_missing_workspace_is_reported(lib):
    a = _args(plan_splits=4)
    assert lib.mamba_selective_scan_fwd(ctypes.byref(a), None) == sss.MSS_ERR_WORKSPACE
    a.workspace = 0x10000
    a.workspace_bytes = 16
    assert lib.mamba_selective_scan_fwd(ctypes.byref(a), None) == sss.MSS_ERR_WORKSPACE


def test_null_args_rejected(lib):
    n = ctypes.c_size_t()
    assert lib.mss_scan_workspace_size(None, ctypes.byref(n)) == sss.MSS_ERR_INVALID_ARG
    assert lib.mamba_selective_scan_fwd(None, None) == sss.MSS_ERR_INVALID_ARG
    assert lib.selective_state_update(None, None) == sss.MSS_ERR_INVALID_ARG
    u = sss.UpdateArgs()
    u.batch, u.dim, u.dstate = 1, 1, 17
    assert lib.selective_state_update(ctypes.byref(u), None) == sss.MSS_ERR_UNSUPPORTED


def _bwd_args(**kw):
    a = sss.ScanBwdArgs()
    a.batch, a.dim, a.dstate, a.seqlen = 2, 40, 16, 1000
    a.in_dtype = sss.MSS_BF16
    fake = 0x10000
    for f in ("u", "delta", "A", "B", "C", "dy", "du", "ddelta", "dA", "dB", "dC"):
        setattr(a, f, fake)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_bwd_workspace_is_two_states_per_block():
    lib = sss.load_library()
    n = ctypes.c_size_t(0)
    assert lib.mss_scan_bwd_workspace_size(ctypes.byref(_bwd_args()), ctypes.byref(n)) == sss.MSS_OK
    # (block start, mid-block) x 2 batch rows x 2 channel tiles x 63 blocks
    # x 16 states x 32 lanes x 4 B
    assert n.value == 2 * 2 * 2 * 63 * 16 * 32 * 4
    # packed sequences keep the block starts only
    a = _bwd_args(cu_seqlens=0x10000, num_seqs=2)
    assert lib.mss_scan_bwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == sss.MSS_OK
    assert n.value == 2 * 2 * 63 * 16 * 32 * 4


@pytest.mark.parametrize("kw,code", [
    (dict(batch=0), sss.MSS_ERR_INVALID_ARG),
    (dict(dstate=17), sss.MSS_ERR_UNSUPPORTED),
    (dict(dy=0), sss.MSS_ERR_INVALID_ARG),
    (dict(dB=0), sss.MSS_ERR_INVALID_ARG),
    (dict(D=0x10000), sss.MSS_ERR_INVALID_ARG),        # D given without dD
    (dict(dz=0x10000), sss.MSS_ERR_INVALID_ARG),       # dz without z
    (dict(u=0x10001), sss.MSS_ERR_INVALID_ARG),        # misaligned bf16
    (dict(dA=0x10002), sss.MSS_ERR_INVALID_ARG),       # misaligned fp32
])
def test_bwd_bad_arguments_are_rejected(kw, code):
    lib = sss.load_library()
    a = _bwd_args(**kw)
    n = ctypes.c_size_t(0)
    assert lib.mss_scan_bwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == code
    assert lib.mamba_selective_scan_bwd(ctypes.byref(a), None) == code


def test_bwd_missing_workspace_is_reported():
    lib = sss.load_library()
    assert lib.mamba_selective_scan_bwd(ctypes.byref(_bwd_args()), None) == sss.MSS_ERR_WORKSPACE


def test_checkpoint_buffer_matches_the_workspace_size():
    """The backward's own sweep keeps the two arrays of states of the
    forward's checkpoint buffer (block starts and mid-block); with the
    forward's checkpoints it needs no workspace here (no device to plan a
    cut schedule for)."""
    lib = sss.load_library()
    for N in (1, 4, 5, 9, 12, 16):
        a = _bwd_args(dstate=N, seqlen=1000)
        n = ctypes.c_size_t(0)
        assert lib.mss_scan_bwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == sss.MSS_OK
        buf = sss.scan_checkpoints(2, 40, N, 1000, "cpu")
        assert buf.numel() * 4 == n.value, N
        a.checkpoints = 256
        assert lib.mss_scan_bwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == sss.MSS_OK
        assert n.value == 0, N


def _ssd_args(**kw):
    a = sss.SsdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.ngroups, a.dstate = 2, 1000, 8, 64, 2, 128
    a.in_dtype, a.out_dtype = sss.MSS_BF16, sss.MSS_F32
    fake = 0x10000
    a.x = a.dt = a.A = a.B = a.C = a.y = fake
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(headdim=32), sss.MSS_ERR_UNSUPPORTED),
    (dict(dstate=64), sss.MSS_ERR_UNSUPPORTED),
    (dict(in_dtype=sss.MSS_F32), sss.MSS_ERR_UNSUPPORTED),
    (dict(ngroups=3), sss.MSS_ERR_INVALID_ARG),
    (dict(seqlen=0), sss.MSS_ERR_INVALID_ARG),
    (dict(batch=0), sss.MSS_ERR_INVALID_ARG),
    (dict(x=0), sss.MSS_ERR_INVALID_ARG),
    (dict(y=0), sss.MSS_ERR_INVALID_ARG),
    (dict(B=0x10008), sss.MSS_ERR_INVALID_ARG),
    (dict(z=0x10004), sss.MSS_ERR_INVALID_ARG),
    (dict(dt=0x10001), sss.MSS_ERR_INVALID_ARG),
    (dict(h0=0x10002), sss.MSS_ERR_INVALID_ARG),
    (dict(in_dtype=7), sss.MSS_ERR_INVALID_ARG),
], ids=lambda v: str(v))
def test_ssd_argument_checks(lib, kw, code):
    """Rejected before anything is enqueued (no GPU is touched)."""
    assert lib.mamba2_ssd_fwd(ctypes.byref(_ssd_args(**kw)), None) == code


@pytest.mark.parametrize("kw", [dict(batch=0), dict(seqlen=0), dict(nheads=0)],
                         ids=lambda v: str(v))
def test_ssd_workspace_size_checks_sizes_first(lib, kw):
    """Bad sizes are rejected before the device is asked for its SM count."""
    n = ctypes.c_size_t(7)
    assert lib.mss_ssd_workspace_size(ctypes.byref(_ssd_args(**kw)), ctypes.byref(n)) == \
        sss.MSS_ERR_INVALID_ARG
    assert lib.mss_ssd_workspace_size(None, ctypes.byref(n)) == sss.MSS_ERR_INVALID_ARG
