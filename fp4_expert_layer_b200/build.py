"""Build the sm_100a shared library in-tree with nvcc.

``libfp4moe.so`` is the product library; ``libfp4moe_checked.so`` is the same
sources with the device bounds checks compiled in (-DMOE_DEBUG_CHECKS): every
index a kernel reads from device data is checked before use and a bad one is
reported through the layer's error word instead of faulting.  The package
loads the checked library when FP4MOE_CHECKED=1 is set in the environment.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
SO = os.path.join(HERE, "libfp4moe.so")
SO_CHECKED = os.path.join(HERE, "libfp4moe_checked.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date(so: str = SO) -> bool:
    if not os.path.exists(so):
        return False
    t = os.path.getmtime(so)
    return all(os.path.getmtime(d) <= t for d in _deps())


def nvcc_cmd(out: str, extra=()):
    return (["nvcc", "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
             "--threads", "0", "-I", INCLUDE, "-I", CSRC, "-o", out] + list(extra) + sources())


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    so = SO_CHECKED if checked else SO
    if not force and up_to_date(so):
        return so
    tmp = so + f".tmp{os.getpid()}"
    extra = (["-Xptxas", "-v"] if verbose else []) + (["-DMOE_DEBUG_CHECKS"] if checked else [])
    subprocess.run(nvcc_cmd(tmp, extra), check=True)
    os.replace(tmp, so)
    return so


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv, checked="--checked" in sys.argv))
