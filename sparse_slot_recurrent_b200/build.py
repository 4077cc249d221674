"""Compile the CUDA sources in ``csrc/`` into ``libramnet.so`` (in-tree, sm_100a only).

nvcc cross-compiles for sm_100a without a GPU.  The CUDA runtime is linked statically,
so the library does not depend on which libcudart the host process (e.g. torch) loads.
``build(debug=True)`` builds ``libramnet_debug.so`` with RAMNET_DEBUG defined: every kernel
then range-checks the slot, ring and event indices it computes and records a failed check
in the status word (ramnet_sync_status reports RAMNET_ERR_DEVICE_CHECK) instead of making
the access.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT = os.path.join(PKG, "libramnet.so")
OUT_DEBUG = os.path.join(PKG, "libramnet_debug.so")
BUILD_DIR = os.path.join(ROOT, "_build")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC",
    "-Xptxas", "-warn-spills",
]


def _nvcc() -> str:
    return shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))


def needs_build(debug: bool = False) -> bool:
    out = OUT_DEBUG if debug else OUT
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in _deps())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Build ``libramnet.so`` (``libramnet_debug.so`` if ``debug``) if any source is newer (or
    ``force``); return its path."""
    out = OUT_DEBUG if debug else OUT
    if not force and not needs_build(debug):
        return out
    bdir = os.path.join(BUILD_DIR, "debug" if debug else "release")
    os.makedirs(bdir, exist_ok=True)
    nvcc = _nvcc()
    flags = NVCC_FLAGS + (["-DRAMNET_DEBUG"] if debug else [])

    def compile_one(src):
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        cmd = [nvcc, *flags, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr)
        return obj

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, _sources()))
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
           "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    import sys
    print(build(force=True, verbose=True, debug="--debug" in sys.argv))
