"""Builds libattn.so in-tree with nvcc for sm_100a (B200).

Usage: python -m exact_tiled_attention_44_b200._build [--verbose]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "attn_api.cu")
DEPS = [os.path.join(PKG, "csrc", f) for f in ("attn_api.cu", "attn_kernel.cuh", "ptx.cuh", "bwd_kernel.cuh",
                                                   "decode_kernel.cuh")] + [
    os.path.join(ROOT, "include", "attn.h")]
OUT = os.path.join(PKG, "libattn.so")


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def flags(verbose: bool = False) -> list[str]:
    f = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
         "-I", os.path.join(PKG, "csrc")]
    if verbose:
        f += ["-Xptxas", "-v"]
    return f


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return OUT
    tmp = OUT + ".tmp"
    cmd = [nvcc_path()] + flags(verbose) + ["-o", tmp, SRC]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
