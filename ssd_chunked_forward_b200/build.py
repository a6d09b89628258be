"""Builds libssd.so (the C-ABI library in csrc/) for sm_100a with nvcc.

    python -m ssd_chunked_forward_b200.build [--verbose-ptxas] [--force]

Objects go to ``_build/`` at the repository root; the library is written next
to this file so it travels with the source tree.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT = os.path.join(PKG, "libssd.so")
BUILD = os.path.join(ROOT, "_build", "libssd")
# the debug variant: every self-addressed global access index-checked
# (SSD_DEBUG_CHECKS), relocatable device code for the one shared record
OUT_DEBUG = os.path.join(PKG, "libssd_debug.so")
BUILD_DEBUG = os.path.join(ROOT, "_build", "libssd_debug")
DEBUG_FLAGS = ["-DSSD_DEBUG_CHECKS", "-rdc=true"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                     "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "kernels", "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "**", "*.cuh"), recursive=True)
                  + glob.glob(os.path.join(CSRC, "**", "*.h"), recursive=True)
                  + glob.glob(os.path.join(ROOT, "include", "*.h")))


def _compile(src: str, verbose_ptxas: bool, debug: bool = False) -> str:
    rel = os.path.relpath(src, CSRC).replace(os.sep, "_")
    obj = os.path.join(BUILD_DEBUG if debug else BUILD, rel + ".o")
    cmd = ([nvcc()] + NVCC_FLAGS + (DEBUG_FLAGS if debug else []) + (["-Xptxas", "-v"] if verbose_ptxas else [])
           + ["-c", src, "-o", obj])
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{res.stdout}\n{res.stderr}")
    if verbose_ptxas:
        sys.stderr.write(res.stderr)
    return obj


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = False) -> str:
    """Build libssd.so, or with debug=True the index-checked libssd_debug.so."""
    out, bdir = (OUT_DEBUG, BUILD_DEBUG) if debug else (OUT, BUILD)
    srcs = sources()
    newest = max(os.path.getmtime(p) for p in srcs + headers() + [__file__])
    if not force and os.path.exists(out) and os.path.getmtime(out) >= newest:
        return out
    os.makedirs(bdir, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose_ptxas, debug), srcs))
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc()] + ARCH + (["-rdc=true"] if debug else []) + ["-shared", "-Xcompiler", "-fPIC", "-o", tmp] + objs
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--debug", action="store_true", help="the index-checked build (libssd_debug.so)")
    args = ap.parse_args()
    print(build(force=args.force, verbose_ptxas=args.verbose_ptxas, debug=args.debug))
