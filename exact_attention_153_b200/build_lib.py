"""Build the sm_100a attention library in-tree: exact_attention_153_b200/libattn_sm100.so.

    python -m exact_attention_153_b200.build_lib [--verbose]

The library is one nvcc translation unit (host API + kernels) compiled for
sm_100a only, with the CUDA runtime linked statically so it works inside any
process that already holds a CUDA context (for example PyTorch's).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libattn_sm100.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)
SOURCES = [os.path.join(CSRC, "attn_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("attn_fwd_sm100.cuh", "sm100_ptx.cuh")] + [
    os.path.join(INCLUDE, "attn.h")]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the sm_100a library cannot be built")


def command(verbose: bool = False) -> list[str]:
    cmd = [
        nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
        "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-O2", "-cudart", "static",
        "-I", INCLUDE, "-I", CSRC, "-o", LIB_PATH, *SOURCES,
    ]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(p) <= t for p in DEPS if os.path.exists(p))


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if a source is newer than it; return its path."""
    if force or verbose or not up_to_date():
        proc = subprocess.run(command(verbose), capture_output=True, text=True)
        if proc.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + proc.stdout + proc.stderr)
        if verbose:
            sys.stderr.write(proc.stdout + proc.stderr)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
