"""Builds librn.so (the CUDA kernels + C ABI) in the package directory.

    python -m rollout_parity_b200.build [--force] [--verbose]

nvcc cross-compiles for sm_100a; no GPU is needed to build.  The flags keep
IEEE arithmetic (no fast math) so the declared rounding order is the executed
one.  Each unit under csrc/ (the host unit rn.cu and one unit per direction and
element format of the row kernels) compiles to an object in a temporary
directory, all at once; the objects are then linked into librn.so.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
SRCS = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
DEPS = SRCS + sorted(glob.glob(os.path.join(CSRC, "*.cuh")))
HDR = os.path.join(ROOT, "include", "rn.h")
LIB = os.path.join(PKG, "librn.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC",
    "--fmad=true", "-prec-div=true", "-prec-sqrt=true", "-ftz=false",
]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found (set NVCC or put the CUDA toolkit on PATH)")


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in (*DEPS, HDR, __file__))


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    inc = ["-I", os.path.join(ROOT, "include"), "-I", CSRC]
    with tempfile.TemporaryDirectory(prefix="rn_build_") as tmpdir:
        procs = []
        for src in SRCS:
            obj = os.path.join(tmpdir, os.path.basename(src)[:-3] + ".o")
            cmd = [nvcc(), *NVCC_FLAGS, *inc, "-c", src, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
                print(" ".join(cmd), flush=True)
            procs.append((src, obj, subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                                     stderr=subprocess.PIPE, text=True)))
        failed = []
        for src, _, p in procs:
            out, err = p.communicate()
            if p.returncode != 0:
                failed.append(src)
                sys.stderr.write(out + err)
            elif verbose:
                sys.stderr.write(err)
        if failed:
            raise RuntimeError(f"nvcc failed building {', '.join(failed)}")
        tmp = LIB + ".tmp"
        cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
               *[o for _, o, _ in procs], "-o", tmp]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"nvcc failed ({r.returncode}) linking {LIB}")
    os.replace(tmp, LIB)
    return LIB


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose))


if __name__ == "__main__":
    main()
