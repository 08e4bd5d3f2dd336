"""The debug build of the library (libkvq_debug.so, -DKVQ_DEBUG): every
kernel checks the global addresses it computes and records a failed check in a
flags word instead of touching memory out of bounds.

CPU: the debug build compiles, loads and exports the same C ABI, reports
itself as the debug build; the normal build refuses kvq_debug_flags.
GPU: small cases of every kernel family run through the debug build (in a
child process, so that it is the library loaded) give the oracle's results
and leave the flags word at 0."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

from quantized_kv_cache_dequantize_b200 import build as kbuild

HERE = os.path.dirname(os.path.abspath(__file__))


def _exports(path):
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    return set(re.findall(r"\bT (kvq_\w+)", out))


def test_debug_build_compiles_and_exports_the_same_abi():
    kbuild.build()
    assert os.path.exists(kbuild.DEBUG_LIB) and os.path.exists(kbuild.LIB)
    assert _exports(kbuild.DEBUG_LIB) == _exports(kbuild.LIB)
    dbg = ctypes.CDLL(kbuild.DEBUG_LIB)
    normal = ctypes.CDLL(kbuild.LIB)
    assert dbg.kvq_debug_build() == 1 and normal.kvq_debug_build() == 0
    normal.kvq_debug_flags.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p]
    word = ctypes.c_uint32(0)
    assert normal.kvq_debug_flags(ctypes.cast(ctypes.byref(word), ctypes.c_void_p), 1, None) == 2  # unsupported
    dbg.kvq_debug_flags.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p]
    assert dbg.kvq_debug_flags(None, 1, None) == 1  # null destination: invalid argument, nothing enqueued


@pytest.mark.gpu
def test_debug_build_runs_every_kernel_family_with_clear_flags(cuda_device):
    kbuild.build()
    env = dict(os.environ, KVQ_DEBUG="1")
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_cases.py")], env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    m = re.search(r"flags=(\d+) checked=(\d+)", r.stdout)
    assert m, r.stdout[-2000:]
    assert int(m.group(1)) == 0, f"debug checks failed: flags {int(m.group(1)):#x}"
    assert int(m.group(2)) >= 17
