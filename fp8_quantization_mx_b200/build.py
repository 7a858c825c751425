"""Builds libmx.so in-tree with nvcc for sm_100a (cross-compiles without a GPU).

    python -m fp8_quantization_mx_b200.build [--force] [--verbose]

Flags: -O3, -lineinfo, IEEE float semantics (no fast math, no flush-to-zero,
IEEE division and square root), static CUDA runtime so that the library loads
on a host without a GPU.
"""

from __future__ import annotations

import argparse
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmx.so")

SOURCES = ["mx_api.cu", "mx_kernels.cu", "mx_bat.cu"]
HEADERS = ["mx_device.cuh", "mx_launch.h", "mx_stream.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
              "-fmad=true", "-Xcompiler", "-fPIC,-O2", "-cudart", "static"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _newest_input() -> float:
    paths = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [os.path.join(INCLUDE, "mx.h"),
                                                                   os.path.abspath(__file__)]
    return max(os.path.getmtime(p) for p in paths)


def build(force: bool = False, verbose: bool = False, extra=None) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= _newest_input():
        return LIB
    # one nvcc per source, in parallel, then one link
    base = [nvcc(), *ARCH, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC]
    if verbose:
        base += ["-Xptxas", "-v"]
    base += list(extra or [])
    objs, procs = [], []
    for src in SOURCES:
        obj = os.path.join(CSRC, src.replace(".cu", ".o"))
        objs.append(obj)
        procs.append((src, subprocess.Popen(base + ["-c", os.path.join(CSRC, src), "-o", obj])))
    failed = [src for src, p in procs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, f"nvcc {' '.join(failed)}")
    subprocess.run([nvcc(), *ARCH, "-shared", "-cudart", "static", *objs, "-o", LIB + ".tmp"],
                   check=True)
    for obj in objs:
        os.remove(obj)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force or args.verbose, verbose=args.verbose), file=sys.stderr)
