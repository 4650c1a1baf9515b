"""Build libbca.so in-tree with nvcc for sm_100a.

    python -m block_causal_attention_dit_b200.build [--verbose]

Static CUDA runtime inside the library (streams are plain driver handles, so the
library works with streams created by any runtime instance, e.g. PyTorch's)."""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libbca.so")
# Self-checking variant (device-side bounds checks, wait-site reporting); used only
# when BCA_LIBRARY points at it.
LIB_CHECKED = os.path.join(PKG, "libbca_checked.so")
# Pipeline-trace variant (clock64 stamps of one CTA's events); BCA_LIBRARY selects it.
LIB_TRACE = os.path.join(PKG, "libbca_trace.so")
SOURCES = [os.path.join(CSRC, "bca.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in
                  ("attn_kernel.cuh", "kv_store_kernel.cuh", "kv_expand_kernel.cuh", "qk_norm_rope_kernel.cuh",
                   "qkv_proj_kernel.cuh",
                   "ulysses_kernel.cuh", "ptx.cuh")] + [
    os.path.join(ROOT, "include", "bca.h")]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str, verbose: bool = False, checked: bool = False, trace: bool = False) -> list:
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
           *(["-DBCA_DEVICE_CHECKS"] if checked else []),
           *(["-DBCA_TRACE"] if trace else []),
           "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared", "-cudart", "static",
           "-I", os.path.join(ROOT, "include"), "-o", out] + SOURCES
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in DEPS)


def build(force: bool = False, verbose: bool = False, checked: bool = False,
          trace: bool = False) -> str:
    lib = LIB_CHECKED if checked else (LIB_TRACE if trace else LIB)
    if not force and up_to_date(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.run(command(tmp, verbose, checked, trace), check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--checked", action="store_true", help="self-checking variant")
    ap.add_argument("--trace", action="store_true", help="pipeline-trace variant")
    a = ap.parse_args()
    print(build(force=True, verbose=a.verbose, checked=a.checked, trace=a.trace))
    sys.exit(0)
