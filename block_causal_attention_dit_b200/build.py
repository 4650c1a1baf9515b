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
SOURCES = [os.path.join(CSRC, "bca.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in
                  ("attn_kernel.cuh", "kv_store_kernel.cuh", "ptx.cuh")] + [
    os.path.join(ROOT, "include", "bca.h")]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str, verbose: bool = False) -> list:
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
           "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared", "-cudart", "static",
           "-I", os.path.join(ROOT, "include"), "-o", out] + SOURCES
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run(command(tmp, verbose), check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=True, verbose=a.verbose))
    sys.exit(0)
