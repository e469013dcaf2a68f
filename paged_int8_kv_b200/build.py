"""Build libkv8.so (the C-ABI CUDA library) in-tree for sm_100a.

    python -m paged_int8_kv_b200.build [--force] [--verbose] [--test-hooks]

Each ``csrc/*.cu`` is compiled by nvcc for ``sm_100a`` and the objects are
linked into ``paged_int8_kv_b200/libkv8.so`` with the CUDA runtime linked
statically, so the library needs nothing at load time beyond the driver.
nvcc cross-compiles, so this runs on a machine without a GPU.

``--test-hooks`` builds ``libkv8_testhooks.so`` instead: the same sources
with ``-DKV8_TEST_HOOKS`` (short bounded waits and the switches declared in
``csrc/kv8_test_hooks.h``), loaded only by the tests of the give-up path.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libkv8.so")
TEST_LIB = os.path.join(HERE, "libkv8_testhooks.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (_sources() + glob.glob(os.path.join(CSRC, "*.cuh")) +
            glob.glob(os.path.join(CSRC, "*.h")) +
            [os.path.join(ROOT, "include", "kv8.h"), __file__])


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in _deps())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          test_hooks: bool = False) -> str:
    lib = TEST_LIB if test_hooks else LIB
    if not force and up_to_date(lib):
        return lib
    bdir = os.path.join(BUILD, "testhooks") if test_hooks else BUILD
    os.makedirs(bdir, exist_ok=True)
    nvcc = _nvcc()
    extra = ["-DKV8_TEST_HOOKS"] if test_hooks else []
    objs = []
    for src in _sources():
        obj = os.path.join(bdir, os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
        if ptxas_info:
            cmd += ["-Xptxas", "-v"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = lib + ".tmp"
    cmd = [nvcc, "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
           "-cudart", "static", "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                ptxas_info="--ptxas-info" in sys.argv,
                test_hooks="--test-hooks" in sys.argv))
