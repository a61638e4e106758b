"""Builds libpagedattn.so in-tree for sm_100a with nvcc.

    python -m paged_kv_cache_361_b200.build [--verbose]

The CUDA runtime is linked statically, so the library loads on a machine
without a GPU (the host block manager works there; device calls report
PA_ERR_CUDA).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libpagedattn.so")

SOURCES = ["capi.cu", "block_manager.cpp", "step.cpp"]
DEPS = ["common.cuh", "cache_ops.cuh", "decode_common.cuh", "decode_simt.cuh", "decode_mma.cuh", "prefill_mma.cuh",
        "tcgen05.cuh", "prefill_tc.cuh", "decode_f8.cuh"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + DEPS] + [os.path.join(INCLUDE, "pagedattn.h"), __file__]
    return [f for f in files if os.path.exists(f)]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def command(out: str = LIB, ptxas_verbose: bool = False, defines=()) -> list[str]:
    """nvcc command line; `defines` are extra -D settings of the kernels'
    build-time tuning knobs (none for the library itself)."""
    cmd = [nvcc(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-Xcompiler", "-fPIC,-O2", "-shared", "-cudart", "static", f"-I{INCLUDE}",
           "-o", out] + [f"-D{d}" for d in defines] + [os.path.join(CSRC, f) for f in SOURCES]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    return cmd


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + ".tmp"
    cmd = command(tmp, ptxas_verbose=verbose)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode:
        raise RuntimeError("nvcc failed building libpagedattn.so")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
