"""Build libattn.so in-tree with nvcc for sm_100a (no JIT cache, so the built library travels with the tree).

libattn_debug.so is the same sources with -DATTN_DEBUG: every plain-address access in the kernels is checked
against its array's extent first (include/attn.h, attn_is_debug_build).

Usage: python -m causal_self_attention_bf16_b200.build [--verbose] [--debug]
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
LIB_PATH = os.path.join(PKG_DIR, "libattn.so")
DEBUG_LIB_PATH = os.path.join(PKG_DIR, "libattn_debug.so")
SOURCES = ["attn_api.cu", "attn_rope.cu"]
DEPENDS = ["attn_api.cu", "attn_rope.cu", "attn_fwd.cuh", "attn_bwd.cuh", "attn_decode.cuh", "attn_common.cuh", "attn_errors.h", "sm100.cuh"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libattn.so")


def command(verbose: bool = False, debug: bool = False):
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=default", "-I", INCLUDE, "-I", CSRC,
           "-o", DEBUG_LIB_PATH if debug else LIB_PATH]
    if debug:
        cmd += ["-DATTN_DEBUG"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    return cmd


def up_to_date(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    deps = [os.path.join(CSRC, d) for d in DEPENDS] + [os.path.join(INCLUDE, "attn.h"), __file__]
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    path = DEBUG_LIB_PATH if debug else LIB_PATH
    if force or not up_to_date(path):
        cmd = command(verbose, debug)
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
        if verbose:
            sys.stdout.write(res.stdout + res.stderr)
    return path


if __name__ == "__main__":
    v = "--verbose" in sys.argv
    print(build(force=True, verbose=v, debug="--debug" in sys.argv))
