"""Build the CUDA library (sm_100a) in-tree: mxfp4_routed_expert_04_b200/libmoe_mxfp4.so.

Usage: python mxfp4_routed_expert_04_b200/build.py [--force] [--verbose-ptxas]
"""
from __future__ import annotations

import argparse
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmoe_mxfp4.so")
BUILD = os.path.join(PKG, "_build")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _inputs_digest() -> str:
    h = hashlib.sha256()
    h.update(" ".join(NVCC_FLAGS).encode())
    files = sources() + sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                               if f.endswith((".h", ".cuh")))
    files.append(os.path.join(os.path.dirname(PKG), "include", "moe_mxfp4.h"))
    for f in files:
        h.update(f.encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def build(force: bool = False, ptxas_verbose: bool = False, jobs: int | None = None,
          out: str | None = None, defines: tuple = ()) -> str:
    """Compile every .cu under csrc/ for sm_100a and link the shared library
    (``out`` and ``defines`` build a variant elsewhere, e.g. for a tuning sweep)."""
    lib = out or LIB
    digest = _inputs_digest() + ",".join(defines)
    stamp = lib + ".sha256"
    if not force and os.path.exists(lib) and os.path.exists(stamp):
        with open(stamp) as f:
            if f.read().strip() == digest:
                return LIB
    bdir = BUILD if out is None else out + ".objs"
    os.makedirs(bdir, exist_ok=True)
    nvcc = _nvcc()
    extra = (["-Xptxas", "-v"] if ptxas_verbose else []) + [f"-D{d}" for d in defines]
    procs, objs = [], []
    for src in sources():
        obj = os.path.join(bdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        cmd = [nvcc, *NVCC_FLAGS, *extra, "-I", CSRC, "-c", src, "-o", obj]
        procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = False
    for cmd, p in procs:
        out, _ = p.communicate()
        text = out.decode(errors="replace")
        if p.returncode != 0:
            failed = True
            sys.stderr.write(" ".join(cmd) + "\n" + text)
        elif ptxas_verbose and text:
            sys.stdout.write(text)
    if failed:
        raise RuntimeError("nvcc failed")
    tmp = lib + ".tmp"
    subprocess.check_call([nvcc, "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-o", tmp, *objs])
    os.replace(tmp, lib)
    with open(stamp, "w") as f:
        f.write(digest)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force or args.verbose_ptxas, ptxas_verbose=args.verbose_ptxas))
