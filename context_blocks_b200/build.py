"""Build ``libpa_attn.so`` in-tree for sm_100a with nvcc.

    python -m context_blocks_b200.build [--verbose]

The library is a single translation unit (``csrc/pa_attn.cu``) that holds the
C ABI of ``include/pa_attn.h`` and both kernels.  The CUDA runtime is linked
statically; the TMA tensor-map encoder is fetched from the driver at run time,
so no link against libcuda is needed and the library cross-compiles on a
machine without a GPU.
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
LIB_PATH = os.path.join(PKG_DIR, "libpa_attn.so")
SOURCES = [os.path.join(CSRC, "pa_attn.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("ptx.cuh", "fwd_common.cuh", "attn_fwd.cuh", "lse_merge.cuh", "quantize.cuh")] + [
    os.path.join(INCLUDE, "pa_attn.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found (CUDA toolkit required to build libpa_attn.so)")
    return cand


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(p) <= t for p in DEPS if os.path.exists(p))


def build(verbose: bool = False, force: bool = False, ptxas_info: bool = False) -> str:
    """Compile the library if any source is newer than it; return its path."""
    if not force and up_to_date():
        return LIB_PATH
    cmd = [_nvcc(), *NVCC_FLAGS, f"-I{INCLUDE}", "-o", LIB_PATH + ".tmp", *SOURCES]
    if ptxas_info:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose or ptxas_info:
        sys.stdout.write(res.stdout + res.stderr)
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    path = build(verbose="--verbose" in sys.argv, force="--force" in sys.argv,
                 ptxas_info="--ptxas-info" in sys.argv)
    print(path)
