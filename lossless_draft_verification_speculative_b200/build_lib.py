"""Build the C-ABI shared library ``libdspark_verify.so`` in-tree for sm_100a.

    python -m lossless_draft_verification_speculative_b200.build_lib

compiles ``csrc/dspark_verify.cu`` (the kernels and their C ABI) and ``csrc/policy.cc`` (the
host-side speculation policy) with nvcc (``-gencode arch=compute_100a,code=sm_100a``),
links the CUDA runtime statically and writes the library next to this file, under
``_lib/``. The Python binding loads it from there.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(PKG_DIR, "_lib")
LIB_PATH = os.path.join(LIB_DIR, "libdspark_verify.so")
SOURCES = ["dspark_verify.cu", "policy.cc"]
HEADERS = ["common.cuh", "stream.cuh", "finish.cuh", "early_exit.cuh", "markov.cuh",
           "markov_mma.cuh"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build the library")


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files += [os.path.join(INCLUDE, h) for h in ("dspark_verify.h", "dspark_policy.h")]
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def nvcc_command(out_path: str = LIB_PATH, extra=()) -> list:
    return [
        nvcc_path(),
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
        "-Xptxas", "-warn-spills",
        "-I", INCLUDE, "-I", CSRC,
        *extra,
        "-o", out_path,
        *[os.path.join(CSRC, s) for s in SOURCES],
    ]


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compile the library unless it is newer than every source. Returns its path."""
    if not force and not extra and up_to_date():
        return LIB_PATH
    os.makedirs(LIB_DIR, exist_ok=True)
    tmp = LIB_PATH + ".tmp"
    cmd = nvcc_command(tmp, extra)
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout, res.stderr, sep="\n", flush=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True,
                extra=("-Xptxas", "-v") if "--ptxas-v" in sys.argv else ()))
