"""Builds libattn.so in-tree with nvcc for sm_100a (no JIT cache, no torch extension).

    python -m exact_attention_sdpa_b200.build [--force] [--verbose] [--debug]

--debug builds libattn_debug.so: the same kernels with their device-side index and range
checks compiled in (status ATTN_ERR_CHECK instead of a fault).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libattn.so")
DEBUG_LIB = os.path.join(PKG, "libattn_debug.so")
SOURCES = [os.path.join(PKG, "csrc", "attn_api.cu")]
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    """The nvcc to use: $NVCC, then the one on PATH, then /usr/local/cuda/bin/nvcc."""
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; set NVCC or put the CUDA toolkit's bin/ on PATH")


def _inputs():
    files = set(SOURCES)
    files.update(glob.glob(os.path.join(PKG, "csrc", "*")))
    files.update(glob.glob(os.path.join(ROOT, "include", "*.h")))
    return sorted(files)


def is_stale(lib: str = LIB) -> bool:
    """True when the library is missing or older than any CUDA source or public header."""
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile libattn.so (or, with debug=True, libattn_debug.so: the device-side index and range
    checks compiled in) in the package directory for sm_100a, when stale or forced; returns its
    path.  Raises RuntimeError with nvcc's output if the compilation fails."""
    out = DEBUG_LIB if debug else LIB
    if not force and not is_stale(out):
        return out
    cmd = [nvcc_path(), *ARCH_FLAGS, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
           "-I" + os.path.join(ROOT, "include"), *(["-DATTN_DEBUG=1"] if debug else []), "-o", out + ".tmp",
           *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        print(res.stdout + res.stderr)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    path = build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv)
    print(path)
