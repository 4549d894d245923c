"""Build libmglu.so in-tree with nvcc for sm_100a.

    python -m masked_glu_b200.build

The library is one translation unit (``csrc/mglu_api.cu`` includes the kernel
headers); the CUDA runtime is linked statically, the driver API is reached
through the runtime's entry-point query, so the shared object loads on a
machine without a GPU (calls then fail with MGLU_ERR_CUDA).
"""
from __future__ import annotations

import glob
import hashlib
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmglu.so")
STAMP = LIB + ".sha256"  # hash of the sources and flags the library was built from
# Test-only build: bounded waits give up after 20 ms and mglu_test_set_stall
# can stop the tensor-core kernel's producer after its first stage, so a test
# can drive the timeout path (the product library has neither).
TEST_LIB = os.path.join(PKG, "libmglu_testhooks.so")
TEST_FLAGS = ["-DMGLU_TEST_HOOKS"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-ldl",
]


def _sources():
    return [os.path.join(CSRC, "mglu_api.cu")]


def _deps():
    return (glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
            + [os.path.join(INCLUDE, "mglu.h")])


def source_hash(extra_flags=()) -> str:
    """SHA-256 over every source the library depends on, the compiler flags
    and the nvcc version: the library is rebuilt whenever any of them
    changes, whatever the files' modification times say."""
    h = hashlib.sha256()
    h.update(" ".join(NVCC_FLAGS + list(extra_flags)).encode())
    h.update(os.environ.get("NVCC", "nvcc").encode())
    try:
        ver = subprocess.run([os.environ.get("NVCC", "nvcc"), "--version"], capture_output=True, text=True).stdout
    except OSError:
        ver = ""
    h.update(ver.encode())
    for p in sorted(_deps()):
        h.update(os.path.relpath(p, ROOT).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def up_to_date(lib: str = LIB, extra_flags=()) -> bool:
    stamp = lib + ".sha256"
    if not (os.path.exists(lib) and os.path.exists(stamp)):
        return False
    with open(stamp) as f:
        return f.read().strip() == source_hash(extra_flags)


def _compile(lib: str, extra_flags, force: bool, verbose: bool) -> str:
    if not force and up_to_date(lib, extra_flags):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, *extra_flags, "-I" + INCLUDE, "-I" + CSRC, "-o", tmp, *_sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    digest = source_hash(extra_flags)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    stamp = lib + ".sha256"
    with open(stamp + ".tmp", "w") as f:
        f.write(digest + "\n")
    os.replace(stamp + ".tmp", stamp)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile csrc/ into masked_glu_b200/libmglu.so (skipped when up to date)."""
    return _compile(LIB, (), force, verbose)


def build_test_hooks(force: bool = False) -> str:
    """Compile the test-hook variant into masked_glu_b200/libmglu_testhooks.so."""
    return _compile(TEST_LIB, TEST_FLAGS, force, False)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
