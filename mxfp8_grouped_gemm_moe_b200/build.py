"""Builds libmxmoe.so in-tree with nvcc for sm_100a (B200), and on request the checked
build libmxmoe_checks.so (-DMXMOE_CHECKS=1: device-side bounds checks that record
MXMOE_ERR_DEVICE_CHECK and skip the access; same API, slower, for tests)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmxmoe.so")
LIB_CHECKS = os.path.join(HERE, "libmxmoe_checks.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")))


def needs_build(lib=LIB):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def nvcc():
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


def build(force=False, verbose=False, ptxas_v=False, checks=False):
    lib = LIB_CHECKS if checks else LIB
    if not force and not needs_build(lib):
        return lib
    cmd = [nvcc()] + NVCC_FLAGS + (["-DMXMOE_CHECKS=1"] if checks else []) + (
        ["-Xptxas", "-v"] if ptxas_v else []) + ["-o", lib + ".tmp", os.path.join(CSRC, "mxmoe_unity.cu")]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if verbose or ptxas_v:
        sys.stderr.write(r.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_v="--ptxas-v" in sys.argv, checks="--checks" in sys.argv)
