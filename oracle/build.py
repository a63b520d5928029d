"""Compile the C++ fp64 oracle (oracle/moe_oracle.cpp) into oracle/libmoe_oracle.so.

Plain g++ (C++17), no fast-math, floating-point contraction off, so every sum
keeps the order the source gives. Rebuilt only when the source or the flags
change (a digest stamp beside the library). Test infrastructure only.

Usage: python oracle/build.py [--force]
"""
from __future__ import annotations

import hashlib
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.cpp")
LIB = os.path.join(HERE, "libmoe_oracle.so")
FLAGS = ["-std=c++17", "-O2", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
         "-fno-fast-math", "-Wall", "-Wextra"]


def _digest() -> str:
    h = hashlib.sha256(" ".join(FLAGS).encode())
    with open(SRC, "rb") as f:
        h.update(f.read())
    return h.hexdigest()


def build(force: bool = False) -> str:
    stamp = LIB + ".sha256"
    dig = _digest()
    if not force and os.path.exists(LIB) and os.path.exists(stamp):
        with open(stamp) as f:
            if f.read().strip() == dig:
                return LIB
    cxx = shutil.which("g++") or shutil.which("c++")
    if not cxx:
        raise RuntimeError("no C++ compiler (g++) to build the oracle")
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call([cxx, *FLAGS, SRC, "-o", tmp])
    os.replace(tmp, LIB)
    with open(stamp, "w") as f:
        f.write(dig)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
