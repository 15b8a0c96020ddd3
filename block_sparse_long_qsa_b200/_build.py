"""Build of libqsa.so (the C-ABI library) from csrc/*.cu for sm_100a, in-tree."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libqsa.so")
BUILD_DIR = os.path.join(PKG, "_build")
# the debug build (tests of the failure handling): the same sources with the
# device bounds checks, the fault-injection hooks of include/qsa_debug.h and
# a 20 ms limit on every device-side wait
LIB_DEBUG = os.path.join(PKG, "libqsa_debug.so")
BUILD_DIR_DEBUG = os.path.join(PKG, "_build_debug")
DEBUG_FLAGS = ["-DQSA_DEBUG_BOUNDS", "-DQSA_DEBUG_HOOKS", "-DQSA_WAIT_TIMEOUT_NS=20000000ull"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2",
    "-I", INCLUDE, "-I", CSRC,
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every csrc/*.cu to an object (in parallel) and link libqsa.so
    (debug=True: libqsa_debug.so with the debug flags)."""
    lib = LIB_DEBUG if debug else LIB
    bdir = BUILD_DIR_DEBUG if debug else BUILD_DIR
    if not force and not _stale(lib):
        return lib
    os.makedirs(bdir, exist_ok=True)
    procs, objs = [], []
    for src in sources():
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        objs.append(obj)
        cmd = ["nvcc", *NVCC_FLAGS, *(DEBUG_FLAGS if debug else []), "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        if out and (verbose or p.returncode != 0):
            sys.stderr.write(out)
        if p.returncode != 0:
            failed.append(src)
    if failed:
        raise RuntimeError(f"nvcc failed for: {failed}")
    subprocess.run(["nvcc", "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs, "-o", lib],
                   check=True)
    return lib


def build_all(force: bool = False) -> tuple[str, str]:
    """The release library and the debug build."""
    return build(force), build(force, debug=True)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
