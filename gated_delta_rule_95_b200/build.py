"""Builds the CUDA library libgdn2.so in-tree with nvcc (sm_100a only)."""
from __future__ import annotations

import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libgdn2.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def deps():
    return sources() + glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + \
        glob.glob(os.path.join(HERE, "csrc", "*.h")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


# The instrumented build (per-chunk clock stamps of the chunk kernel, GDN2_STAMPS) goes to a
# library of its own, never loaded by the package unless a profiling run asks for it.
LIB_STAMPS = os.path.join(HERE, "libgdn2_stamps.so")


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in deps())


def build(force: bool = False, verbose: bool = False, stamps: bool = False) -> str:
    """Compile every .cu under csrc/ into one shared library; returns its path.  stamps=True
    builds the instrumented variant (libgdn2_stamps.so) instead."""
    lib = LIB_STAMPS if stamps else LIB
    if not force and up_to_date(lib):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    objs = []
    bdir = os.path.join(HERE, "_build", "stamps" if stamps else "")
    os.makedirs(bdir, exist_ok=True)
    for src in sources():
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        cmd = [nvcc, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
               "-I", os.path.join(ROOT, "include"), "-c", src, "-o", obj]
        if stamps:
            cmd.insert(1, "-DGDN2_STAMPS")
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.run(cmd, check=True)
        objs.append(obj)
    subprocess.run([nvcc, *ARCH, "-shared", *objs, "-o", lib], check=True)
    return lib


if __name__ == "__main__":
    import sys
    print(build(force=True, verbose="-v" in sys.argv, stamps="--stamps" in sys.argv))
