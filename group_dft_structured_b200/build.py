"""Builds libfeql.so (the CUDA library behind include/feql.h) in-tree for sm_100a.

    python -m group_dft_structured_b200.build [--verbose]

nvcc cross-compiles without a GPU; the .so lands next to this file.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libfeql.so")
# Failure-detection test build: a 20 ms bound on every device-side wait and one
# accumulator-release arrive left out of the forward kernel, so that a bounded
# wait runs out (tests/test_wait_timeout_gpu.py).  Not for use outside tests.
TIMEOUT_LIB = os.path.join(PKG, "libfeql_waittest.so")
TIMEOUT_FLAGS = ["-DFEQL_WAIT_LIMIT_NS=20000000ull", "-DFEQL_TEST_SKIP_FIRST_RELEASE=1"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2",
    "--expt-relaxed-constexpr",
    "-shared",
]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return [os.path.join(CSRC, "feql_api.cu")]


def deps() -> list[str]:
    out = [os.path.join(ROOT, "include", "feql.h")]
    for f in os.listdir(CSRC):
        if f.endswith((".cu", ".cuh")):
            out.append(os.path.join(CSRC, f))
    return out


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in deps())


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          lib: str = LIB) -> str:
    if not force and up_to_date(lib):
        return lib
    cmd = [nvcc(), *NVCC_FLAGS, *(extra or []), "-o", lib + ".tmp", *sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose:
        print(r.stdout + r.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


def build_waittest(force: bool = False) -> str:
    """The failure-detection test library (see TIMEOUT_LIB)."""
    return build(force=force, extra=TIMEOUT_FLAGS, lib=TIMEOUT_LIB)


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
