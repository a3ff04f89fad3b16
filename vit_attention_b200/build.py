"""Build libvggt_attn.so in-tree for sm_100a (B200).

    python vit_attention_b200/build.py [--force] [--debug]

(Run as a file, not through the package: the package's __init__ loads the
library this script builds.)

nvcc cross-compiles without a GPU.  The CUDA runtime is linked statically, so
the library only needs the NVIDIA driver at run time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libvggt_attn.so")
LIB_DEBUG = os.path.join(HERE, "libvggt_attn_debug.so")   # -DVGGT_DEBUG: device-side bounds checks
SOURCES = [os.path.join(HERE, "csrc", "vggt_attn.cu")]
DEPENDS = SOURCES + sorted(os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc"))
                           if f.endswith(".cuh")) + [os.path.join(ROOT, "include", "vggt_attn.h")]
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or put the CUDA 12.9 toolkit on PATH)")


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in DEPENDS)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Build the release library, or with debug=True the debug build (libvggt_attn_debug.so: -DVGGT_DEBUG,
    device-side bounds checks that record VGGT_ATTN_ERR_BOUNDS instead of faulting)."""
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(lib):
        return lib
    cmd = [nvcc(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xptxas", "-v", "-I", os.path.join(ROOT, "include"), *(["-DVGGT_DEBUG"] if debug else []),
           "-o", lib + ".tmp", *SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stderr}")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
