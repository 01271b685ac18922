"""Build the CUDA library libvcattn.so in-tree for sm_100a with nvcc.

    python -m bit_fp8_attention_smooth_b200.build [--force] [--verbose]

The library is a plain shared object exporting the C ABI of
include/vc_attention.h; it links the CUDA runtime statically and reaches the
driver (tensor-map encoding) through cudaGetDriverEntryPoint, so it needs no
libcuda at link time.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libvcattn.so")


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libvcattn.so")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [os.path.join(INCLUDE, "vc_attention.h")]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in deps())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + f".{os.getpid()}.tmp"
    cmd = [
        nvcc(), "-shared", "-Xcompiler", "-fPIC", "-std=c++17", "-O3", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        # IEEE fp32 throughout: the ExpCast byte map reads a rounded integer
        # out of an fp32 subnormal, so denormals must not be flushed; divisions
        # and square roots are the correctly rounded ones the quantisers use.
        # (--use_fast_math would turn all three off, so it is never passed.)
        "--ftz=false", "--prec-div=true", "--prec-sqrt=true",
        "--expt-relaxed-constexpr", "-Xptxas", "-v" if verbose else "-O3",
        "-I", INCLUDE, "-I", CSRC,
        "-o", tmp, *sources(),
    ]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        print(res.stdout)
        print(res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode})")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
