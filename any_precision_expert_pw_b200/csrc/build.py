"""Build libpw in-tree with nvcc for sm_100a (one translation unit, static cudart): libpw.so,
and libpw_debug.so, the same sources with PW_DEBUG (device bounds checks that record
PW_ERR_BOUNDS instead of touching memory outside a buffer)."""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
ROOT = os.path.dirname(PKG)
OUT = os.path.join(PKG, "libpw.so")
OUT_DEBUG = os.path.join(PKG, "libpw_debug.so")
OUT_CEILING = os.path.join(PKG, "decode_ceiling")
SOURCES = [os.path.join(HERE, "pw_lib.cu")]
DEPS = [os.path.join(HERE, f) for f in os.listdir(HERE) if f.endswith((".cu", ".cuh"))] + [
    os.path.join(ROOT, "include", "pw.h")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def command(verbose_ptxas: bool = False, debug: bool = False):
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-O2", "-cudart", "static",
           "-I", os.path.join(ROOT, "include"), "-o", OUT_DEBUG if debug else OUT] + SOURCES
    if debug:
        cmd.insert(1, "-DPW_DEBUG")
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def up_to_date(out: str) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = True) -> str:
    """Build libpw.so (and libpw_debug.so unless debug=False) when out of date; returns the
    path of libpw.so.  The two compile in parallel."""
    jobs = [(OUT, False)] + ([(OUT_DEBUG, True)] if debug else [])
    todo = [(out, dbg) for out, dbg in jobs if force or verbose_ptxas or not up_to_date(out)]
    with ThreadPoolExecutor(max_workers=2) as ex:
        for f in [ex.submit(subprocess.run, command(verbose_ptxas, dbg), check=True)
                  for _, dbg in todo]:
            f.result()
    return OUT


def build_ceiling() -> str:
    """The decode-ceiling measurement program (decode_ceiling.cu, a standalone executable)."""
    subprocess.run([nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
                    "-std=c++17", "-I", os.path.join(ROOT, "include"), "-I", HERE, "-o",
                    OUT_CEILING, os.path.join(HERE, "decode_ceiling.cu")], check=True)
    return OUT_CEILING


if __name__ == "__main__":
    if "--ceiling" in sys.argv:
        print(build_ceiling())
    else:
        build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv)
        print(OUT)
