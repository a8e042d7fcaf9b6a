"""Build libattn_b200.so in-tree with nvcc (sm_100a only).

Usage: ``python -m attention_tiled_exact_b200.build [--force] [--verbose] [--debug]``.
The library lands next to this file, so it travels with the source tree.
``--debug`` builds the bounds-checking libattn_b200_debug.so instead.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libattn_b200.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)
# The same sources with ATTN_DEBUG_BOUNDS=1: every kernel checks its shared-
# memory, tensor-memory and output indices before the access.
DEBUG_LIB_NAME = "libattn_b200_debug.so"
DEBUG_LIB_PATH = os.path.join(HERE, DEBUG_LIB_NAME)

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libattn_b200.so")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> list[str]:
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def is_stale(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every .cu under csrc/ into one shared library; returns its path.

    debug=True builds the bounds-checking variant (ATTN_DEBUG_BOUNDS=1)."""
    path = DEBUG_LIB_PATH if debug else LIB_PATH
    if not force and not is_stale(path):
        return path
    tmp = path + ".tmp"
    defs = ["-DATTN_DEBUG_BOUNDS=1"] if debug else []
    cmd = [_nvcc(), *NVCC_FLAGS, *defs, "-I", INCLUDE, "-I", CSRC, "-shared", "-o", tmp, *sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose:
        sys.stdout.write(res.stdout + res.stderr)
    os.replace(tmp, path)
    return path


def ensure_built() -> str:
    return build(force=False)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
