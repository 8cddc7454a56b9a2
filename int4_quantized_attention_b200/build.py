"""Build the C-ABI library librotate_attn.so in-tree with nvcc for sm_100a,
and its test build librotate_attn_bounds.so (every computed global index
checked before use, a violation reported through the device error word)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "librotate_attn.so")
LIB_BOUNDS = os.path.join(PKG, "librotate_attn_bounds.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
    "-shared", "-cudart", "static",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                  + glob.glob(os.path.join(ROOT, "include", "*.h")))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in sources() + headers() + [__file__])


def _compile(lib: str, extra, verbose: bool) -> subprocess.Popen:
    cmd = [NVCC, *NVCC_FLAGS, *extra, "-I", os.path.join(ROOT, "include")]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-o", lib + ".tmp", *sources()]
    return subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)


def build(force: bool = False, verbose: bool = False, bounds: bool = True) -> str:
    """Compile every .cu under csrc/ into the shared library (and, with
    bounds=True, the bounds-checked test build, in parallel); returns the
    production library's path."""
    jobs = []
    if force or not up_to_date(LIB):
        jobs.append((LIB, _compile(LIB, [], verbose)))
    if bounds and (force or not up_to_date(LIB_BOUNDS)):
        jobs.append((LIB_BOUNDS, _compile(LIB_BOUNDS, ["-DRA_BOUNDS_CHECK=1"], verbose)))
    failed = []
    for lib, proc in jobs:
        out, err = proc.communicate()
        if proc.returncode != 0:
            sys.stderr.write(out + err)
            failed.append(os.path.basename(lib))
        else:
            if verbose:
                sys.stderr.write(err)
            os.replace(lib + ".tmp", lib)
    if failed:
        raise RuntimeError("nvcc failed building " + ", ".join(failed))
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
