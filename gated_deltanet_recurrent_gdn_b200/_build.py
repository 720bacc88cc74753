"""Build of the CUDA library ``libgdn.so`` (in-tree, sm_100a only)."""
from __future__ import annotations

import os
import shutil
import subprocess

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
REPO_DIR = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(REPO_DIR, "include")
LIB_PATH = os.path.join(PKG_DIR, "libgdn.so")
SOURCES = [os.path.join(CSRC, "gdn_api.cu")]
DEPS = SOURCES + [
    os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cuh", ".h"))
] + [os.path.join(INCLUDE, "gdn.h")]

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xcompiler", "-fvisibility=hidden",
]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libgdn.so")


def stale(lib_path: str = LIB_PATH) -> bool:
    if not os.path.exists(lib_path):
        return True
    t = os.path.getmtime(lib_path)
    return any(os.path.getmtime(d) > t for d in DEPS)


# A test build of the library for the timeout branches of the bounded waits:
# the waits give up after 200 us instead of a second, and the waits of the
# multi-token block form and of the low-rank kernel expect 16 bytes more
# than their bulk copy delivers, so they run out without any fault.  Only
# tests load it.
WAIT_TEST_LIB_PATH = os.path.join(PKG_DIR, "libgdn_waittest.so")
WAIT_TEST_DEFINES = ("GDN_WAIT_LIMIT_NS=200000ull", "GDN_WAIT_TEST_EXTRA_TX=16u")


def build_library(force: bool = False, out: str = LIB_PATH, defines=(), verbose: bool = False) -> str:
    """Compile ``csrc/gdn_api.cu`` into ``out`` with nvcc for sm_100a.

    ``defines`` are extra ``NAME=VALUE`` preprocessor definitions (the test
    build's wait settings, launch shape overrides).  An existing ``out`` is
    rebuilt only when a source is newer or ``force`` is set.  The library
    links the CUDA runtime statically and exports only the ``gdn_*`` C
    symbols."""
    if not force and not stale(out):
        return out
    tmp = f"{out}.tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC]
    cmd += [f"-D{d}" for d in defines]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-o", tmp, *SOURCES]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build_wait_test_library(force: bool = False) -> str:
    """The test build described at WAIT_TEST_DEFINES."""
    return build_library(force=force, out=WAIT_TEST_LIB_PATH, defines=WAIT_TEST_DEFINES)
