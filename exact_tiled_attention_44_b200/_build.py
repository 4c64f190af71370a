"""Builds libattn.so in-tree with nvcc for sm_100a (B200).

The library is five translation units (shared host code, the forward for
d <= 64, the forward for d = 128, the backward, decode), compiled in parallel
to objects under ``_objs/`` and linked into ``libattn.so``.

Usage: python -m exact_tiled_attention_44_b200._build [--verbose]
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
UNITS = ["attn_api.cu", "fwd_api.cu", "fwd_d128.cu", "bwd_api.cu", "decode_api.cu"]
HEADERS = [os.path.join(CSRC, f) for f in ("host.h", "fwd_launch.cuh", "attn_kernel.cuh", "ptx.cuh", "bwd_kernel.cuh",
                                           "decode_tc_kernel.cuh")] + [os.path.join(ROOT, "include", "attn.h")]
DEPS = [os.path.join(CSRC, u) for u in UNITS] + HEADERS
OUT = os.path.join(PKG, "libattn.so")
OBJ_DIR = os.path.join(PKG, "_objs")


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def flags(verbose: bool = False) -> list[str]:
    f = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"), "-I", CSRC]
    if verbose:
        f += ["-Xptxas", "-v"]
    return f


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def _run(cmd: list[str]) -> subprocess.CompletedProcess:
    return subprocess.run(cmd, capture_output=True, text=True)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return OUT
    os.makedirs(OBJ_DIR, exist_ok=True)
    nvcc = nvcc_path()
    cmds = [[nvcc] + flags(verbose) + ["-c", "-o", os.path.join(OBJ_DIR, u[:-3] + ".o"),
                                       os.path.join(CSRC, u)] for u in UNITS]
    with cf.ThreadPoolExecutor(max_workers=len(cmds)) as ex:
        results = list(ex.map(_run, cmds))
    for cmd, res in zip(cmds, results):
        if res.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
        if verbose:
            sys.stderr.write(res.stdout + res.stderr)
    tmp = OUT + ".tmp"
    link = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp] + \
        [os.path.join(OBJ_DIR, u[:-3] + ".o") for u in UNITS]
    res = _run(link)
    if res.returncode != 0:
        raise RuntimeError("nvcc link failed:\n" + " ".join(link) + "\n" + res.stdout + res.stderr)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
