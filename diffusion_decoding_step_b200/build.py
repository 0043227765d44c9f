"""Build libdllm.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libdllm.so")
# The same sources with DLLM_DEBUG: row positions read from device memory are
# range-checked in the kernels (an error bit instead of an access).
LIB_DEBUG = os.path.join(HERE, "libdllm_debug.so")
SOURCES = ["api.cu", "gemm.cu", "attn.cu", "small.cu", "stack.cu"]
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps.append(os.path.join(HERE, "..", "include", "dllm.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every CUDA source into libdllm.so next to this file (with
    debug=True: libdllm_debug.so, the DLLM_DEBUG build)."""
    lib = LIB_DEBUG if debug else LIB
    if not force and not stale(lib):
        return lib
    cmd = [nvcc(), *FLAGS]
    if debug:
        cmd += ["-DDLLM_DEBUG"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    tmp = lib + ".tmp"
    cmd += ["-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                debug="--debug" in sys.argv))
