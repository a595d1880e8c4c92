"""Build libpoetx.so (the POET-X layer's C ABI and its sm_100a kernels) in
place, next to this file, with nvcc; `debug=True` builds libpoetx_debug.so,
the same library compiled with -DPOETX_DEBUG (every TMA and bulk copy checked
before it is issued; see csrc/ptx.cuh), loaded instead when the environment
sets POETX_DEBUG=1."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libpoetx.so")
LIB_DEBUG = os.path.join(HERE, "libpoetx_debug.so")
SOURCES = ["poetx.cu"]


def deps():
    return (sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))) +
            [os.path.join(ROOT, "include", "poetx.h")])


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(d) > t for d in deps() if os.path.exists(d))


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not needs_build(lib):
        return lib
    cmd = [nvcc(), "-std=c++17", "-O3", "-lineinfo", "-gencode", "arch=compute_100a,code=sm_100a",
           "-shared", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           "-o", lib + ".tmp"] + [os.path.join(CSRC, s) for s in SOURCES] + ["-lcudart"]
    if debug:
        cmd.insert(1, "-DPOETX_DEBUG")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
