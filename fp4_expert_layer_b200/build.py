"""Build the sm_100a shared library ``libfp4moe.so`` in-tree with nvcc."""
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
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date() -> bool:
    if not os.path.exists(SO):
        return False
    t = os.path.getmtime(SO)
    return all(os.path.getmtime(d) <= t for d in _deps())


def nvcc_cmd(out: str, extra=()):
    return (["nvcc", "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
             "--threads", "0", "-I", INCLUDE, "-I", CSRC, "-o", out] + list(extra) + sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return SO
    tmp = SO + f".tmp{os.getpid()}"
    extra = ["-Xptxas", "-v"] if verbose else []
    subprocess.run(nvcc_cmd(tmp, extra), check=True)
    os.replace(tmp, SO)
    return SO


if __name__ == "__main__":
    build(force=True, verbose="-v" in sys.argv)
    print(SO)
