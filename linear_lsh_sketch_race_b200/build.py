"""Build librace_attn.so in place with nvcc for sm_100a.

Usage: python -m linear_lsh_sketch_race_b200.build [--verbose-ptxas] [--bounds-check]

--bounds-check builds librace_attn_checked.so instead: the same library compiled with
-DRACE_BOUNDS_CHECK, whose kernels test their data-dependent indices (bucket ids of the
hard-hash path, the per-plane gradient rows of the backward sweeps), skip an access out of
range and raise the bounds bit of the device status flag.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "librace_attn.so")
LIB_CHECKED = os.path.join(PKG, "librace_attn_checked.so")
SOURCES = ["race_attn.cu"]


def nvcc_cmd(ptxas_verbose: bool = False, out: str = LIB, bounds_check: bool = False):
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
    if bounds_check:
        cmd.insert(1, "-DRACE_BOUNDS_CHECK")
    return cmd


def newest_source_mtime() -> float:
    paths = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    paths.append(os.path.join(ROOT, "include", "race_attn.h"))
    paths.append(os.path.abspath(__file__))
    return max(os.path.getmtime(p) for p in paths)


def build(force: bool = False, ptxas_verbose: bool = False, bounds_check: bool = False) -> str:
    lib = LIB_CHECKED if bounds_check else LIB
    if (not force and os.path.exists(lib)
            and os.path.getmtime(lib) >= newest_source_mtime()):
        return lib
    tmp = lib + ".tmp"
    subprocess.run(nvcc_cmd(ptxas_verbose, tmp, bounds_check), check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv,
                bounds_check="--bounds-check" in sys.argv))
