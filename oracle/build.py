"""Builds the oracle's shared library with the host compiler (no CUDA)."""

from __future__ import annotations

import hashlib
import os
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))


def oracle_library_path() -> str:
    return os.path.join(_HERE, "libmx_oracle.so")


def build_oracle(force: bool = False) -> str:
    """Compiles the oracle unless the library in place was built from this
    exact source and command (recorded hash; file times are not trusted)."""
    src = os.path.join(_HERE, "mx_oracle.cpp")
    out = oracle_library_path()
    cmd = ["g++", "-O2", "-std=c++17", "-Wall", "-Wextra", "-shared", "-fPIC", "-pthread",
           "-ffp-contract=off", src, "-o", out + ".tmp"]
    with open(src, "rb") as f:
        want = hashlib.sha256(f.read() + " ".join(cmd[:-3]).encode()).hexdigest()
    stamp = out + ".srchash"
    have = open(stamp).read().strip() if os.path.exists(stamp) else ""
    if not force and os.path.exists(out) and have == want:
        return out
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    with open(stamp, "w") as f:
        f.write(want + "\n")
    return out


if __name__ == "__main__":
    print(build_oracle(force=True))
