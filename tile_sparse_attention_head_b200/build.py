"""Builds the in-tree CUDA library libveda.so for sm_100a with nvcc.

The library is one translation unit (csrc/veda_api.cu includes the kernel
sources) linked against the static CUDA runtime; the driver API entry point
it needs (cuTensorMapEncodeTiled) is fetched at run time, so no -lcuda.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libveda.so")
# Debug build: every computed index is checked in the kernels (-DVEDA_DEBUG_BOUNDS);
# a failed check is reported by veda_sync_status as VEDA_ERR_BOUNDS.  The
# binding loads it instead of LIB when VEDA_DEBUG_BOUNDS=1 is set.
DEBUG_LIB = os.path.join(HERE, "libveda_debug.so")
SOURCES = ["veda_api.cu", "veda_common.cuh", "kernels.h", "permute_tripool.cu", "score_topk.cu",
           "sparse_attn.cu", "tile_map.cu", "estimator.cu", "distill.cu", "attn_bwd.cu"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def nvcc_command(out: str = LIB, extra=()) -> list:
    return [nvcc_path(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
            "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr", *extra,
            "-o", out, os.path.join(CSRC, "veda_api.cu")]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + [os.path.join(HERE, "..", "include", "veda.h")]
    return all(os.path.getmtime(p) <= t for p in deps if os.path.exists(p))


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    if not force and up_to_date(lib):
        return lib
    tmp = lib + ".tmp"
    extra = (["-Xptxas", "-v"] if verbose else []) + (["-DVEDA_DEBUG_BOUNDS"] if debug else [])
    cmd = nvcc_command(tmp, extra)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, lib)
    return lib


def build_all(force: bool = False) -> list:
    """The release library and the debug (bounds-checked) one, compiled side by side."""
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(2) as ex:
        futs = [ex.submit(build, force, False, dbg) for dbg in (False, True)]
        return [f.result() for f in futs]


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
