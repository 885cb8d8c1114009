"""Builds libsolattn.so in-tree for sm_100a with nvcc.

    python -m block_sparse_attention_cov_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsolattn.so")
# Test-only variant (failure-detection tests): adds solattn_test_set_hook, which
# makes one CTA skip its first K tile and shortens the bounded-wait budget.
LIB_HOOKS = os.path.join(PKG, "libsolattn_testhooks.so")
SOURCES = ["api.cu", "pool.cu", "forward.cu", "forward_pp.cu"]
HEADERS = ["kernels.h", "ptx.cuh", "fwd_common.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libsolattn.so")


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "solattn.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, hooks: bool = False) -> str:
    """Compiles the library (or, with hooks, its test-hook variant) if a source
    is newer than it (or force); returns its path."""
    lib = LIB_HOOKS if hooks else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + ".tmp"
    extra = ["-DSOLATTN_TEST_HOOKS"] if hooks else []
    cmd = [_nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, "-o", tmp] + [os.path.join(CSRC, f) for f in SOURCES]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + proc.stdout + proc.stderr)
    if verbose:
        sys.stderr.write(proc.stdout + proc.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
    print(build(force="--force" in sys.argv, hooks=True))
