"""Build the CUDA library in-tree: csrc/*.cu -> libfa_b200.so (sm_100a only).

Run ``python -m tiled_exact_attention_forward_b200.build`` (or call
:func:`build`).  The compiler is nvcc from CUDA 12.9; nothing is JIT-compiled
at import time, and the built library sits next to this file so it travels
with the source tree.

Each source is compiled to an object of its own (in parallel) as whole-program
device code -- one module per source file, no device linking: under separate
compilation (-rdc) ptxas ignores the per-warpgroup register budgets that the
forward kernel sets with setmaxnreg -- then one nvcc call links them.  Flags can differ per file: the
float32 forward (the exact path of the single-head fp32 workload) is built
without ``--use_fast_math`` so its exp2, log and division are the IEEE-rounded
ones; every other kernel calls its fast instructions explicitly and keeps the
fast-math flags it was measured with.
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ_DIR = os.path.join(HERE, "_build")
LIB_NAME = "libfa_b200.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON_FLAGS = [
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-I", os.path.join(ROOT, "include"),
]
FAST_MATH = ["--use_fast_math"]
# Sources built with IEEE-rounded float32 math (no --use_fast_math).
EXACT_MATH_SOURCES = {"fwd_f32.cu"}


def nvcc() -> str:
    cand = [os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"]
    for c in cand:
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found: the CUDA 12.9 toolkit is required to build the library")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def flags_for(src: str):
    """nvcc flags of one source file."""
    name = os.path.basename(src)
    return [*ARCH_FLAGS, *COMMON_FLAGS, *([] if name in EXACT_MATH_SOURCES else FAST_MATH)]


def _inputs():
    files = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    files += glob.glob(os.path.join(ROOT, "include", "*.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def _compile(src: str, extra, verbose: bool):
    obj = os.path.join(OBJ_DIR, os.path.basename(src)[:-3] + ".o")
    cmd = [nvcc(), *flags_for(src), *(extra or []), "-c", "-o", obj, src]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, cwd=CSRC, capture_output=True, text=True)
    return obj, r


def build(force: bool = False, verbose: bool = False, extra_flags=None) -> str:
    """Compile every kernel for sm_100a into libfa_b200.so; returns its path."""
    if not force and up_to_date():
        return LIB_PATH
    os.makedirs(OBJ_DIR, exist_ok=True)
    srcs = sources()
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(len(srcs), os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda s: _compile(s, extra_flags, verbose), srcs))
    objs = []
    for (obj, r), src in zip(results, srcs):
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)} with exit code {r.returncode}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr)
        objs.append(obj)
    tmp = LIB_PATH + ".tmp"
    cmd = [nvcc(), *ARCH_FLAGS, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, cwd=CSRC, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc link failed with exit code {r.returncode}")
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    v = "-v" in sys.argv
    flags = ["-Xptxas", "-v"] if "--ptxas" in sys.argv else None
    print(build(force="--force" in sys.argv, verbose=v or bool(flags), extra_flags=flags))
