"""Build libwq_b200.so in-tree with nvcc for sm_100a.

Flags that matter for the numerics: -fmad=false (no multiply is fused into a following add, so
every fp32 step rounds as the pages' PyTorch code does) and the default IEEE division and square
root (no fast-math). The CUDA runtime is linked statically so that the library does not depend
on which libcudart the host process loaded.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libwq_b200.so")
BUILD_DIR = os.path.join(PKG, "_build")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")) + glob.glob(os.path.join(PKG, "csrc", "*.cpp")))


def _deps():
    return sources() + glob.glob(os.path.join(PKG, "csrc", "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in _deps())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    common = ["-O3", "-std=c++17", "-lineinfo", "-fmad=false", "-Xcompiler", "-fPIC,-O2,-ffp-contract=off",
              "-I", os.path.join(ROOT, "include"), "-I", os.path.join(PKG, "csrc")] + ARCH
    if verbose:
        common += ["-Xptxas", "-v"]
    # an object is reused when it is newer than its source and every header (and this script)
    headers = [h for h in _deps() if not h.endswith((".cu", ".cpp"))] + [os.path.abspath(__file__)]
    newest_header = max(os.path.getmtime(h) for h in headers)
    objs = []
    for src in sources():
        obj = os.path.join(BUILD_DIR, os.path.basename(src) + ".o")
        fresh = (not force and os.path.exists(obj) and
                 os.path.getmtime(obj) > max(os.path.getmtime(src), newest_header))
        if not fresh:
            subprocess.run([NVCC, "-c", src, "-o", obj] + common, check=True)
        objs.append(obj)
    tmp = LIB + ".tmp"
    subprocess.run([NVCC, "-shared", "-o", tmp] + objs + ARCH + ["-cudart", "static", "-Xlinker", "--no-undefined"],
                   check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
