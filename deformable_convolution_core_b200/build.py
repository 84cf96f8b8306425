"""Build the CUDA library in-tree: libdcncore.so next to this file.

nvcc compiles the single translation unit csrc/dcn_core.cu for sm_100a only
(the library has no other target) with the C ABI of include/dcn_core.h.
Fast-math is deliberately off: the softmax uses expf and the sampling
location must be rounded exactly as the operator's contract states.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libdcncore.so")
# The bounds-checked build: every global access of the kernels is tested
# against its tensor's extent first (a substitute for a memory checker).
LIB_CHECKED = os.path.join(HERE, "libdcncore_checked.so")
SOURCES = [os.path.join(CSRC, "dcn_core.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(INCLUDE, "dcn_core.h")]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def nvcc_command(out: str, extra: list[str] | None = None) -> list[str]:
    return [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
            "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
            "-I", INCLUDE, "-o", out] + (extra or []) + SOURCES


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(d) > t for d in DEPS)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    """Build libdcncore.so (or, with checked=True, libdcncore_checked.so with
    -DDCN_CHECK_BOUNDS) next to this file, if a source is newer."""
    lib = LIB_CHECKED if checked else LIB
    if force or needs_build(lib):
        tmp = lib + ".tmp.%d" % os.getpid()
        extra = (["-Xptxas", "-v"] if verbose else []) + (["-DDCN_CHECK_BOUNDS"] if checked else [])
        res = subprocess.run(nvcc_command(tmp, extra), capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
        if verbose:
            sys.stderr.write(res.stderr)
        os.replace(tmp, lib)
    return lib


def build_all(force: bool = False) -> list[str]:
    """Build the library and its bounds-checked twin side by side (two nvcc
    processes; each is one translation unit)."""
    from concurrent.futures import ThreadPoolExecutor

    with ThreadPoolExecutor(2) as ex:
        jobs = [ex.submit(build, force, False, c) for c in (False, True)]
        return [j.result() for j in jobs]


if __name__ == "__main__":
    if "--all" in sys.argv:
        print(build_all(force="--force" in sys.argv))
    else:
        print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                    checked="--checked" in sys.argv))
