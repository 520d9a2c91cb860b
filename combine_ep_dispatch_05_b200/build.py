"""Build libep_b200.so in-tree with nvcc for sm_100a.

    python -m combine_ep_dispatch_05_b200.build [--force]
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libep_b200.so")
# The bounds-checking build: every copy's addresses are checked against their
# buffers' extents, and an access outside is skipped and reported
# (EP_DEVERR_BOUNDS) instead of made. Load it with EP_B200_LIBRARY=debug.
LIB_DEBUG = os.path.join(PKG, "libep_b200_debug.so")
SOURCES = [os.path.join(PKG, "csrc", "ep_abi.cu"), os.path.join(PKG, "csrc", "ep_kernels.cu"),
           os.path.join(PKG, "csrc", "ep_noalloc.cu"), os.path.join(PKG, "csrc", "ep_comm.cu")]
DEPS = SOURCES + glob.glob(os.path.join(PKG, "csrc", "*.h")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-I" + os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libep_b200.so")


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(d) > t for d in DEPS)


OBJ_DIR = os.path.join(ROOT, "_build")


def _objects(lib: str, extra: list, verbose: bool) -> list:
    """(object path, compile command) of every source of `lib`."""
    tag = os.path.splitext(os.path.basename(lib))[0]
    jobs = []
    for src in SOURCES:
        obj = os.path.join(OBJ_DIR, f"{tag}.{os.path.splitext(os.path.basename(src))[0]}.{os.getpid()}.o")
        cmd = [nvcc(), *NVCC_FLAGS, *extra, "-c", "-o", obj, src]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        jobs.append((obj, cmd))
    return jobs


def build(force: bool = False, verbose: bool = False) -> str:
    """Build the library and its bounds-checking twin (every translation unit
    compiled in parallel, then linked); return the library's path."""
    from concurrent.futures import ThreadPoolExecutor
    libs = [(lib, extra) for lib, extra in ((LIB, []), (LIB_DEBUG, ["-DEP_DEBUG_BOUNDS"]))
            if force or stale(lib)]
    if not libs:
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    plan = [(lib, _objects(lib, extra, verbose and lib == LIB)) for lib, extra in libs]
    cmds = [cmd for _, jobs in plan for _, cmd in jobs]
    with ThreadPoolExecutor(max_workers=min(len(cmds), os.cpu_count() or 1)) as pool:
        for rc, cmd in zip(pool.map(lambda c: subprocess.run(c).returncode, cmds), cmds):
            if rc != 0:
                raise subprocess.CalledProcessError(rc, cmd)
    for lib, jobs in plan:
        tmp = lib + f".tmp{os.getpid()}"
        objs = [o for o, _ in jobs]
        subprocess.check_call([nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs])
        os.replace(tmp, lib)
        for o in objs:
            os.remove(o)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
