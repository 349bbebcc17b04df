"""Builds liblitela.so in-tree for sm_100a with nvcc.

    python -m linear_attention_diffusion_litela_b200.build

The library is a plain shared object with a C ABI (include/litela.h); it links the CUDA
runtime only (the driver API entry points it needs are fetched at run time), so it loads on
a machine without a GPU.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
LIB_PATH = os.path.join(PKG_DIR, "liblitela.so")
SOURCES = ["litela_abi.cu"]
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or put the CUDA toolkit on PATH")


def build(verbose: bool = False, extra_flags=None) -> str:
    """Compile every CUDA source into liblitela.so; returns the library path."""
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "litela.h")]
    if os.path.exists(LIB_PATH) and not extra_flags:
        lib_mtime = os.path.getmtime(LIB_PATH)
        if all(os.path.getmtime(p) <= lib_mtime for p in deps):
            return LIB_PATH
    cmd = [nvcc_path(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "--shared",
           "-Xcompiler", "-fPIC,-O2", "-cudart", "shared", "-Xptxas", "-v" if verbose else "-O3",
           "-I", os.path.join(ROOT, "include"),
           *(extra_flags or []),
           "-o", LIB_PATH + ".tmp", *[os.path.join(CSRC, s) for s in SOURCES]]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed (%d):\n%s\n%s" % (res.returncode, " ".join(cmd), res.stderr))
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
