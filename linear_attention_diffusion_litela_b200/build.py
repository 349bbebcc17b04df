"""Builds liblitela.so (and the benchmark's liblitela_ffma_peak.so) in-tree for sm_100a with nvcc.

    python -m linear_attention_diffusion_litela_b200.build

The libraries are plain shared objects with a C ABI (include/litela.h,
include/litela_ffma_peak.h); they link the CUDA runtime only (the driver API entry points
liblitela needs are fetched at run time), so they load on a machine without a GPU.
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
PEAK_DIR = os.path.join(PKG_DIR, "peaks")
FFMA_LIB_PATH = os.path.join(PKG_DIR, "liblitela_ffma_peak.so")
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or put the CUDA toolkit on PATH")


def _nvcc_shared(out, sources, deps, verbose, extra_flags):
    if os.path.exists(out) and not extra_flags:
        lib_mtime = os.path.getmtime(out)
        if all(os.path.getmtime(p) <= lib_mtime for p in deps):
            return out
    cmd = [nvcc_path(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "--shared",
           "-Xcompiler", "-fPIC,-O2", "-cudart", "shared", "-Xptxas", "-v" if verbose else "-O3",
           "-I", os.path.join(ROOT, "include"),
           *(extra_flags or []),
           "-o", out + ".tmp", *sources]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed (%d):\n%s\n%s" % (res.returncode, " ".join(cmd), res.stderr))
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(out + ".tmp", out)
    return out


def build(verbose: bool = False, extra_flags=None) -> str:
    """Compile every CUDA source: liblitela.so (the method) and liblitela_ffma_peak.so (the
    benchmark's FMA-peak measurement); returns liblitela's path."""
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "litela.h")]
    _nvcc_shared(LIB_PATH, [os.path.join(CSRC, s) for s in SOURCES], deps, verbose, extra_flags)
    peak_src = os.path.join(PEAK_DIR, "ffma_peak.cu")
    _nvcc_shared(FFMA_LIB_PATH, [peak_src], [peak_src, os.path.join(ROOT, "include", "litela_ffma_peak.h")],
                 verbose, extra_flags)
    return LIB_PATH


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
