"""Build libsvdq.so (the CUDA library behind include/svdq.h) in-tree with nvcc
for sm_100a.  Usage: python -m diffusion_transformer_w4a4_b200.build"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsvdq.so")
# the bounds-checked debug variant: same sources with -DSVDQ_DEBUG_BOUNDS
LIB_DEBUG = os.path.join(HERE, "libsvdq_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(HERE, "..", "include", "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None, debug: bool = False) -> str:
    """Compile libsvdq.so (or, with debug=True, libsvdq_debug.so: every kernel's
    self-addressed global accesses bounds-checked, errors in the status word)."""
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    if debug:
        extra = list(extra or []) + ["-DSVDQ_DEBUG_BOUNDS"]
    nvcc = os.environ.get("NVCC", "nvcc")
    objdir = os.path.join(HERE, "_build_debug" if debug else "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    procs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [nvcc, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-ffp-contract=off",
               "--fmad=false" if src.endswith("host_prepare.cpp") else "--fmad=true",
               "-I", os.path.join(HERE, "..", "include"), "-c", src, "-o", obj, *(extra or [])]
        if src.endswith(".cpp"):
            cmd = [nvcc, *ARCH, "-O3", "-std=c++17", "-Xcompiler", "-fPIC,-ffp-contract=off,-pthread",
                   "-I", os.path.join(HERE, "..", "include"), "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        procs.append(subprocess.Popen(cmd))
        objs.append(obj)
    bad = [p.args for p in procs if p.wait() != 0]
    if bad:
        raise RuntimeError(f"nvcc failed for: {[b[-3] for b in bad]}")
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call([nvcc, *ARCH, "-shared", "-o", tmp, *objs, "-lpthread"])
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
