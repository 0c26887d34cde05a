"""Build libjmoe.so (the C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libjmoe.so")
CHECKS_LIB = os.path.join(HERE, "libjmoe_checks.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_flags(extra=()):
    return ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                   "--expt-relaxed-constexpr", *extra]


def build(verbose: bool = False, ptxas_info: bool = False, checks: bool = False) -> str:
    """Compile every csrc/*.cu to an object, then link libjmoe.so (static cudart).
    checks=True builds libjmoe_checks.so instead: the same sources with the
    device bounds checks compiled in (-DJMOE_CHECKS=1), objects in _build_checks."""
    objdir = os.path.join(HERE, "_build_checks" if checks else "_build")
    lib = CHECKS_LIB if checks else LIB
    os.makedirs(objdir, exist_ok=True)
    objs = []
    extra = (["-Xptxas", "-v"] if ptxas_info else []) + (["-DJMOE_CHECKS=1"] if checks else [])
    for src in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        cmd = ["nvcc", *nvcc_flags(extra), "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    cmd = ["nvcc", *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", lib, *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    return lib


if __name__ == "__main__":
    build(verbose=True, ptxas_info="--ptxas" in sys.argv, checks="--checks" in sys.argv)
