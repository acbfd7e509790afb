"""Build librace_attn.so in place with nvcc for sm_100a.

Usage: python -m linear_lsh_sketch_race_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "librace_attn.so")
SOURCES = ["race_attn.cu"]


def nvcc_cmd(ptxas_verbose: bool = False, out: str = LIB):
    cmd = [
        os.environ.get("NVCC", "nvcc"),
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC,-O2", "-shared",
        "-I", os.path.join(ROOT, "include"), "-I", CSRC,
        "-o", out,
    ] + [os.path.join(CSRC, s) for s in SOURCES]
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def newest_source_mtime() -> float:
    paths = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    paths.append(os.path.join(ROOT, "include", "race_attn.h"))
    paths.append(os.path.abspath(__file__))
    return max(os.path.getmtime(p) for p in paths)


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= newest_source_mtime()):
        return LIB
    tmp = LIB + ".tmp"
    subprocess.run(nvcc_cmd(ptxas_verbose, tmp), check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv))
