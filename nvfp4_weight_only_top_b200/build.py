"""Builds the in-tree shared libraries with nvcc for sm_100a.

  libmoe_nvfp4.so   the MoE layer (csrc/*.cu, C ABI in include/moe_nvfp4.h)
  libmoe_inputs.so  the device writer of synthetic banks (moe_inputs/fill.cu)

Usage: python -m nvfp4_weight_only_top_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
INCLUDE = os.path.join(ROOT, "include")
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmoe_nvfp4.so")
INPUTS_SRC = os.path.join(ROOT, "moe_inputs", "fill.cu")
INPUTS_LIB = os.path.join(ROOT, "moe_inputs", "libmoe_inputs.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(out: str, deps: list) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd: list, log: str, verbose: bool) -> None:
    r = subprocess.run(cmd, capture_output=True, text=True)
    with open(log, "w") as f:
        f.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed ({r.returncode}): {' '.join(cmd)}")
    if verbose:
        sys.stdout.write(r.stdout + r.stderr)


def build(force: bool = False, verbose: bool = False) -> list:
    """Compiles both libraries if their sources changed; returns the library paths."""
    nvcc = _nvcc()
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    deps = srcs + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + glob.glob(os.path.join(INCLUDE, "*.h"))
    if force or _stale(LIB, deps):
        tmp = LIB + ".tmp"
        _run([nvcc, *ARCH, *FLAGS, "-rdc=true", "-I", INCLUDE, "-o", tmp, *srcs],
             os.path.join(PKG, "build_moe_nvfp4.log"), verbose)
        os.replace(tmp, LIB)
    if force or _stale(INPUTS_LIB, [INPUTS_SRC]):
        tmp = INPUTS_LIB + ".tmp"
        _run([nvcc, *ARCH, *FLAGS, "-o", tmp, INPUTS_SRC],
             os.path.join(PKG, "build_moe_inputs.log"), verbose)
        os.replace(tmp, INPUTS_LIB)
    return [LIB, INPUTS_LIB]


if __name__ == "__main__":
    print("\n".join(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)))
