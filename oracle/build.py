"""Builds the oracle's shared library with the host compiler (no CUDA)."""

from __future__ import annotations

import os
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))


def oracle_library_path() -> str:
    return os.path.join(_HERE, "libmx_oracle.so")


def build_oracle(force: bool = False) -> str:
    src = os.path.join(_HERE, "mx_oracle.cpp")
    out = oracle_library_path()
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    cmd = ["g++", "-O2", "-std=c++17", "-Wall", "-Wextra", "-shared", "-fPIC", "-pthread",
           "-ffp-contract=off", src, "-o", out]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build_oracle(force=True))
