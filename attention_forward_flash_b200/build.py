"""Builds the CUDA library ``libattn.so`` in-tree with nvcc for sm_100a.

Usage: ``python -m attention_forward_flash_b200.build`` (or ``build()``).
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libattn.so")
SOURCES = [os.path.join(HERE, "csrc", "attn_api.cu")]
DEPS = SOURCES + [os.path.join(HERE, "csrc", f) for f in (
    "ptx.cuh", "flash_fwd.cuh", "quant.cuh", "merge.cuh", "rope.cuh", "decode.cuh",
    "device_once.h")] + [
    os.path.join(os.path.dirname(HERE), "include", "attn.h")]


def nvcc_path():
    p = shutil.which("nvcc")
    if p:
        return p
    cand = "/usr/local/cuda/bin/nvcc"
    if os.path.exists(cand):
        return cand
    raise RuntimeError("nvcc not found")


def needs_build():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(d) > t for d in DEPS)


def build(force=False, verbose=False):
    if not force and not needs_build():
        return LIB
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-o", LIB + ".tmp"] + SOURCES
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
