"""Build libqi21.so in-tree with nvcc for sm_100a.

    python -m prefix_kv_cached_b200.build [-v] [--debug]

--debug builds libqi21_debug.so instead, with QI21_DEBUG defined: every
kernel launch is followed by a stream synchronisation and an error check that
names the kernel that failed (outside stream capture). Load it by setting
QI21_LIB to its path before importing the binding.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libqi21.so")
DEBUG_LIB = os.path.join(HERE, "libqi21_debug.so")
SOURCES = ["qi21_api.cu", "qi21_noalloc.cu", "qi21_host.cpp"]
HEADERS = ["qi21_internal.h", "qi21_common.cuh", "qi21_simt.cuh", "qi21_sm100.cuh", "qi21_gemm_tc.cuh",
           "qi21_attn_tc.cuh", "qi21_final_tc.cuh"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "qi21.h")]
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def build(verbose: bool = False, force: bool = False, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    if not force and not needs_build(lib):
        return lib
    cmd = [
        _nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v" if verbose else "-O3",
        "-I", os.path.join(ROOT, "include"), "-I", CSRC,
        "-o", lib,
    ] + (["-DQI21_DEBUG"] if debug else []) + [os.path.join(CSRC, s) for s in SOURCES]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if verbose:
        sys.stderr.write(r.stderr)
    return lib


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force=True, debug="--debug" in sys.argv))
