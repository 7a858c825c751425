"""Builds libmx.so in-tree with nvcc for sm_100a (cross-compiles without a GPU).

    python -m fp8_quantization_mx_b200.build [--force] [--verbose]

Flags: -O3, -lineinfo, IEEE float semantics (no fast math, no flush-to-zero,
IEEE division and square root), static CUDA runtime so that the library loads
on a host without a GPU.
"""

from __future__ import annotations

import argparse
import hashlib
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmx.so")

SOURCES = ["mx_api.cu", "mx_kernels.cu", "mx_bat.cu", "mx_gemm.cu"]
HEADERS = ["mx_device.cuh", "mx_launch.h", "mx_stream.cuh", "mx_tc.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
              "-fmad=true", "-Xcompiler", "-fPIC,-O2", "-cudart", "static"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


STAMP = LIB + ".srchash"


def source_hash(extra=None) -> str:
    """SHA-256 over every source, header and flag the library is built from."""
    h = hashlib.sha256()
    paths = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [os.path.join(INCLUDE, "mx.h"),
                                                                   os.path.abspath(__file__)]
    for p in paths:
        h.update(os.path.basename(p).encode() + b"\0")
        with open(p, "rb") as f:
            h.update(f.read())
    h.update(" ".join(ARCH + NVCC_FLAGS + list(extra or [])).encode())
    return h.hexdigest()


def _stamp() -> str:
    try:
        with open(STAMP) as f:
            return f.read().strip()
    except OSError:
        return ""


def build(force: bool = False, verbose: bool = False, extra=None) -> str:
    """Builds libmx.so unless the one in place was built from these exact
    sources and flags (its recorded source hash matches); file times are not
    trusted, so a stale library is always rebuilt."""
    want = source_hash(extra)
    if not force and not verbose and os.path.exists(LIB) and _stamp() == want:
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
    with open(STAMP + ".tmp", "w") as f:
        f.write(want + "\n")
    os.replace(STAMP + ".tmp", STAMP)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force or args.verbose, verbose=args.verbose), file=sys.stderr)
