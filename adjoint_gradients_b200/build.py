"""Build libqml.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m adjoint_gradients_b200.build [--force] [--debug]

The shared library lands next to this file so it travels with the source tree.
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
LIB = os.path.join(HERE, "libqml.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra=None) -> str:
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h*")) + [os.path.join(INCLUDE, "qml.h"), __file__]
    if not force and not _stale(LIB, deps):
        return LIB
    cmd = [
        "nvcc", *ARCH, "-lineinfo", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
        "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC,
        "-DQML_BUILD", "--expt-relaxed-constexpr",
        *sources(), "-o", LIB + ".tmp", "-lcudart",
    ]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    if extra:
        cmd[1:1] = list(extra)
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
