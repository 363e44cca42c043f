"""Build libkvq.so in-tree with nvcc for sm_100a (B200).

    python -m int8_quantized_paged_quantize_b200.build [--verbose-ptxas]

Objects go to ``_build/`` at the repository root; the shared library is written
next to this file so it travels with the package. The C-ABI library links the
CUDA runtime statically and has no PyTorch dependency.
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libkvq.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3", "-I", INCLUDE, "-I", CSRC]
SOURCES = ["kvq_kernels.cu", "kvq_api.cpp", "kvq_pool.cpp", "kvq_noalloc.cu"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _run(cmd):
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
        raise RuntimeError(f"build step failed: {os.path.basename(cmd[-1])}")
    return r.stdout + r.stderr


def _stale(out, deps):
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose_ptxas: bool = False, force: bool = False) -> str:
    """Compile every source and link libkvq.so. Returns the library path."""
    os.makedirs(BUILD, exist_ok=True)
    headers = [os.path.join(INCLUDE, "kvq.h")] + [
        os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    objs = []
    log = []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(BUILD, src + ".o")
        objs.append(obj)
        if force or verbose_ptxas or _stale(obj, [path] + headers):
            extra = ["-Xptxas", "-v"] if (verbose_ptxas and src.endswith(".cu")) else []
            log.append(_run([nvcc()] + ARCH + COMMON + extra + ["-c", "-o", obj, path]))
    if force or _stale(LIB, objs):
        tmp = LIB + ".tmp"
        _run([nvcc()] + ARCH + ["-shared", "-o", tmp] + objs + ["-lcudart_static", "-ldl", "-lrt",
                                                                 "-lpthread"])
        os.replace(tmp, LIB)
    if verbose_ptxas:
        sys.stdout.write("".join(log))
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(a.verbose_ptxas, a.force))


if __name__ == "__main__":
    main()
