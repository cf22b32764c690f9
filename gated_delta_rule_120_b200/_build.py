"""Build libkda.so (the KDA C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libkda.so")
# the bounds-checked build (-DKDA_BOUNDS_CHECK): every global access of the prefill, decode and
# recurrent-mode kernels is tested against the extent of its buffer (a debugging substitute for a
# memory checker); load it with KDA_LIBRARY=<path> before importing the package
LIB_CHECKED = os.path.join(PKG, "libkda_checked.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O3,-fvisibility=hidden",
    "-shared",
    "--expt-relaxed-constexpr",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(CSRC, "*.h")) +
                  glob.glob(os.path.join(ROOT, "include", "*.h")))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    """Compile csrc/kda_lib.cu into gated_delta_rule_120_b200/libkda.so (no-op when current);
    with ``checked`` the bounds-checked build libkda_checked.so instead."""
    lib = LIB_CHECKED if checked else LIB
    if not force and up_to_date(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *NVCC_FLAGS, *(["-DKDA_BOUNDS_CHECK"] if checked else []),
           "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           "-o", tmp, os.path.join(CSRC, "kda_lib.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                checked="--checked" in sys.argv))
