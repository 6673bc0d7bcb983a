"""Build libopr.so (the CUDA library behind include/opr.h) for sm_100a, in-tree.

    python -m block_sparse_masked_segment_b200.build [--verbose] [--force]

nvcc cross-compiles without a GPU.  The shared libraries land next to this
file so that they travel with the source tree:

- ``lib/libopr.so``        the release library;
- ``lib/libopr_debug.so``  the same sources built with ``-DOPR_DEBUG_CHECKS``: the
  attention kernels check the indices they take from the layout tables and set
  OPR_DEV_BOUNDS instead of using a bad one.  The binding loads it when the
  environment sets ``OPR_DEBUG_CHECKS=1``.
"""

from __future__ import annotations

import argparse
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB_DIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIB_DIR, "libopr.so")
LIB_DEBUG = os.path.join(LIB_DIR, "libopr_debug.so")
SOURCES = ["api.cu", "layout.cu", "rope.cu", "attn_fwd.cu", "attn_bwd.cu", "noalloc.cu", "duplicate.cu", "loss.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def nvcc_flags(verbose: bool = False) -> list[str]:
    flags = [
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
        "--expt-relaxed-constexpr",
        "-I", os.path.join(ROOT, "include"),
    ]
    if verbose:
        flags += ["-Xptxas", "-v"]
    return flags


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    inc = os.path.join(ROOT, "include")
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(inc, f) for f in os.listdir(inc)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Build the release library (or, with debug=True, the bounds-checking one); returns its path."""
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    os.makedirs(LIB_DIR, exist_ok=True)
    objs = []
    extra = ["-DOPR_DEBUG_CHECKS"] if debug else []
    for src in SOURCES:
        obj = os.path.join(LIB_DIR, src.replace(".cu", "_debug.o" if debug else ".o"))
        cmd = [NVCC, *nvcc_flags(verbose), *extra, "-c", os.path.join(CSRC, src), "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0 or verbose:
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}")
        objs.append(obj)
    tmp = lib + ".tmp"
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs, "-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"link of {os.path.basename(lib)} failed")
    os.replace(tmp, lib)
    for o in objs:
        os.remove(o)
    return lib


def build_all(force: bool = False) -> list[str]:
    """Both libraries: release and debug checks."""
    return [build(force=force), build(force=force, debug=True)]


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/shared-memory reports")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force or a.verbose, verbose=a.verbose))
    print(build(force=a.force, debug=True))
