"""Build libgdn.so (all CUDA sources, sm_100a) in-tree next to this file.

Usage: ``python -m gated_delta_rule_112_b200.build [--force] [--verbose] [--checked]``.
nvcc cross-compiles for sm_100a without a GPU present. ``--checked`` builds
libgdn_checked.so instead: the same library with device-side bounds checks
(-DGDN_CHECKS=1), the stand-in for a memory checker; it is never the default.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC_DIR = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libgdn.so")
LIB_CHECKED = os.path.join(HERE, "libgdn_checked.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC,-O2",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return sorted(glob.glob(os.path.join(SRC_DIR, "*.cu")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(SRC_DIR, "*.cuh")) + [
        os.path.join(ROOT, "include", "gdn.h"), __file__]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    if not force and not _stale(lib):
        return lib
    obj_dir = os.path.join(HERE, "_build_checked" if checked else "_build")
    os.makedirs(obj_dir, exist_ok=True)
    objs = []
    for src in sources():
        obj = os.path.join(obj_dir, os.path.basename(src) + ".o")
        cmd = [NVCC, *NVCC_FLAGS, *(["-DGDN_CHECKS=1"] if checked else []), "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        objs.append(obj)
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                           *objs, "-o", tmp])
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                checked="--checked" in sys.argv))
