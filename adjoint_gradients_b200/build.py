"""Build libqml.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m adjoint_gradients_b200.build [--force] [-v]

Every source file is compiled to an object of its own, in parallel, under
``_build/``; the objects are then linked into one shared library that lands
next to this file, so it travels with the source tree.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libqml.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = [
    "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-I", INCLUDE, "-I", CSRC, "-DQML_BUILD", "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def headers():
    # every header any source includes (.h, .hpp, .cuh): a change rebuilds every object
    hs = []
    for pat in ("*.h", "*.hpp", "*.cuh"):
        hs += glob.glob(os.path.join(CSRC, pat))
    return hs + [os.path.join(INCLUDE, "qml.h"), __file__]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _obj(src):
    return os.path.join(OBJ_DIR, os.path.basename(src) + ".o")


def build(force: bool = False, verbose: bool = False, extra=None) -> str:
    srcs = sources()
    hdrs = headers()
    if not force and not _stale(LIB, srcs + hdrs):
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    extra = list(extra or [])

    def compile_one(src):
        obj = _obj(src)
        if not force and not _stale(obj, [src] + hdrs):
            return ""
        cmd = ["nvcc", *extra, *ARCH, *FLAGS, "-c", src, "-o", obj + ".tmp"]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}{r.stderr}")
        os.replace(obj + ".tmp", obj)
        return r.stdout + r.stderr

    with ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as pool:
        for out in pool.map(compile_one, srcs):
            if out and verbose:
                sys.stderr.write(out)
    link = ["nvcc", *ARCH, "-shared", *[_obj(s) for s in srcs], "-o", LIB + ".tmp", "-lcudart"]
    subprocess.check_call(link)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
