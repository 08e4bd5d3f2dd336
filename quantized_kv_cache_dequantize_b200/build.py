"""Build libkvq.so (and its debug build, libkvq_debug.so) in-tree with nvcc
for sm_100a.

    python -m quantized_kv_cache_dequantize_b200.build [--verbose] [--debug-only]

The shared libraries are written next to this file so that they travel with
the source tree; they export only the extern "C" entry points of
include/kvq.h.  The debug build is compiled with -DKVQ_DEBUG: its kernels
check every global address they compute and record failures in a flags word
(kvq_debug_flags) instead of touching memory out of bounds.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libkvq.so")
DEBUG_LIB = os.path.join(HERE, "libkvq_debug.so")
SOURCES = [os.path.join(CSRC, "kvq.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + [
    os.path.join(INCLUDE, "kvq.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    # the score-only instantiations of the attention item return before its
    # merge code, which the front end then reports as unreachable
    "-diag-suppress=128",
    "-shared",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in DEPS)


def _command(lib: str, tmp: str, verbose: bool):
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-o", tmp, *SOURCES, "-lcudart"]
    if lib == DEBUG_LIB:
        cmd.insert(1, "-DKVQ_DEBUG")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def build(force: bool = False, verbose: bool = False, debug: bool | None = None) -> str:
    """Compile what is out of date: the normal library (debug False), the
    debug build (debug True), or both at once (debug None, the default: two
    nvcc processes side by side).  Returns the normal library's path (the
    debug one's when debug is True)."""
    libs = [LIB, DEBUG_LIB] if debug is None else [DEBUG_LIB if debug else LIB]
    todo = [lib for lib in libs if force or not up_to_date(lib)]
    procs = []
    for lib in todo:
        tmp = lib + f".tmp{os.getpid()}"
        procs.append((lib, tmp, subprocess.Popen(_command(lib, tmp, verbose))))
    failed = [lib for lib, tmp, pr in procs if pr.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, f"nvcc ({', '.join(os.path.basename(f) for f in failed)})")
    for lib, tmp, _ in procs:
        os.replace(tmp, lib)
    return DEBUG_LIB if debug else LIB


if __name__ == "__main__":
    only_debug = "--debug-only" in sys.argv
    print(build(force=True, verbose="--verbose" in sys.argv, debug=True if only_debug else None))
