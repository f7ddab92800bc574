"""Builds libflashblock.so in-tree with nvcc for sm_100a.

    python -m block_diffusion_attention_b200.build [--force] [--verbose]

Each .cu under csrc/ is compiled to an object under _build/ (rebuilt when it
or any header is newer) and linked into block_diffusion_attention_b200/
libflashblock.so with the CUDA runtime linked statically, so the library
loads on machines without a GPU (its compute entry points then return
FB_ERR_LAUNCH).

The same sources are also built as libflashblock_testhooks.so (objects under
_build/testhooks/) with FB_TEST_HOOKS and a 2 ms bound on every pipeline wait:
a test-only library whose extra entry point fb_test_set_skip_k1 makes the
attention kernels leave one K load out, so the tests can make a wait run out
and check that the time-out is reported and the next call runs normally.
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libflashblock.so")
TEST_LIB = os.path.join(PKG, "libflashblock_testhooks.so")
TEST_DEFS = ["-DFB_TEST_HOOKS", "-DFB_WAIT_LIMIT_NS=2000000ull"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _build_one(lib: str, objdir: str, defs, force: bool, verbose: bool, ptxas_verbose: bool) -> str:
    os.makedirs(objdir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr_mtime = max((os.path.getmtime(h) for h in _headers()), default=0.0)
    objs = []
    relink = force or not os.path.exists(lib)
    for src in srcs:
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if (not force and os.path.exists(obj) and os.path.getmtime(obj) >= os.path.getmtime(src)
                and os.path.getmtime(obj) >= hdr_mtime):
            continue
        cmd = [nvcc()] + ARCH + FLAGS + list(defs) + (["-Xptxas", "-v"] if ptxas_verbose else []) + \
            ["-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        relink = True
    if not relink and all(os.path.getmtime(lib) >= os.path.getmtime(o) for o in objs):
        return lib
    tmp = lib + ".tmp"
    cmd = [nvcc()] + ARCH + ["-shared", "-o", tmp] + objs + ["-cudart", "static"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False, test_lib: bool = True) -> str:
    """Builds libflashblock.so (and, unless test_lib is False, the test-only
    libflashblock_testhooks.so); returns the library's path."""
    out = _build_one(LIB, BUILD, [], force, verbose, ptxas_verbose)
    if test_lib:
        _build_one(TEST_LIB, os.path.join(BUILD, "testhooks"), TEST_DEFS, force, verbose, False)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    a = ap.parse_args(argv)
    print(build(a.force, a.verbose, a.ptxas_verbose))


if __name__ == "__main__":
    sys.exit(main())
