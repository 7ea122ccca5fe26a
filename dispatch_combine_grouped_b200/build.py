"""Build libmoe.so (all CUDA sources, sm_100a) in-tree with nvcc.

    python dispatch_combine_grouped_b200/build.py [--verbose-ptxas]

This file does not import the package (whose import loads the library), so it can run
before the library exists.  Other code loads it by path with ``load_builder()``.
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libmoe.so")
LIB_CHECKED = os.path.join(HERE, "libmoe_checked.so")  # -DMOE_CHECKS: device bounds checks
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h")))


def up_to_date(checked: bool = False) -> bool:
    lib = LIB_CHECKED if checked else LIB
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in sources() + headers() + [__file__])


def build(force: bool = False, ptxas_verbose: bool = False, checked: bool = False) -> str:
    """libmoe.so, or with checked=True the bounds-checked libmoe_checked.so (-DMOE_CHECKS)."""
    lib = LIB_CHECKED if checked else LIB
    if not force and up_to_date(checked):
        return lib
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC,-O2", "-shared", "-I", os.path.join(ROOT, "include"),
           "-o", lib + ".tmp"] + (["-DMOE_CHECKS=1"] if checked else []) + sources()
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv, checked="--checked" in sys.argv)
    print(LIB_CHECKED if "--checked" in sys.argv else LIB)


def load_builder():
    """This module, loaded by file path (without importing the package)."""
    return sys.modules[__name__]
