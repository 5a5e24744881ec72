"""Build the CUDA library libsss48.so in-tree with nvcc (sm_100a only).

``python -m selective_state_space_48_b200.builder`` or ``build()`` compiles
``csrc/*.cu`` into ``_lib/libsss48.so``.  nvcc cross-compiles, so this runs
on a host without a GPU.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(PKG, "_lib")
LIB_PATH = os.path.join(LIB_DIR, "libsss48.so")
DEBUG_LIB_PATH = os.path.join(LIB_DIR, "libsss48_debug.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
              "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc",
                 shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(path: str) -> bool:
    if not os.path.exists(path):
        return True
    mtime = os.path.getmtime(path)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]
    return any(os.path.getmtime(p) > mtime for p in deps)


def _compile(src: str, obj: str, extra: list[str]) -> subprocess.CompletedProcess:
    cmd = [nvcc(), *ARCH_FLAGS, *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC,
           "-c", "-o", obj, src]
    return subprocess.run(cmd, capture_output=True, text=True)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every ``csrc/*.cu`` to an object (in parallel, one nvcc per
    file) and link them into the shared library.  ``debug`` builds the
    checked variant (``MSS_DEBUG``: device-side bounds checks that record
    an error in the status word) into ``_lib/libsss48_debug.so``."""
    out = DEBUG_LIB_PATH if debug else LIB_PATH
    if not force and not _stale(out):
        return out
    from concurrent.futures import ThreadPoolExecutor
    os.makedirs(LIB_DIR, exist_ok=True)
    objdir = os.path.join(LIB_DIR, f"obj{'_debug' if debug else ''}.{os.getpid()}")
    os.makedirs(objdir, exist_ok=True)
    extra = ["-DMSS_DEBUG=1"] if debug else []
    srcs = sources()
    objs = [os.path.join(objdir, os.path.basename(s) + ".o") for s in srcs]
    try:
        with ThreadPoolExecutor(max_workers=min(len(srcs), os.cpu_count() or 4)) as ex:
            results = list(ex.map(lambda so: _compile(so[0], so[1], extra), zip(srcs, objs)))
        for src, res in zip(srcs, results):
            if res.returncode != 0:
                raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n"
                                   f"{res.stdout}\n{res.stderr}")
            if verbose and (res.stdout or res.stderr):
                print(os.path.basename(src), res.stdout, res.stderr)
        tmp = out + f".tmp{os.getpid()}"
        cmd = [nvcc(), *ARCH_FLAGS, "-shared", "-o", tmp, *objs]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"nvcc link failed:\n{res.stdout}\n{res.stderr}")
        os.replace(tmp, out)
    finally:
        shutil.rmtree(objdir, ignore_errors=True)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
