"""Builds libpkvq.so (sm_100a) in-tree with nvcc.

    python -m paged_quantized_kv_quant_b200.build [--force] [--bounds-check]

The library links the CUDA runtime statically and exports only the C ABI of
include/pkvq.h.  ``--bounds-check`` builds ``libpkvq_checked.so`` with
PKVQ_BOUNDS_CHECK, whose kernels skip (and record) block ids and slots that
fall outside the pool instead of reading or writing out of bounds.
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
LIB = os.path.join(PKG, "libpkvq.so")
LIB_CHECKED = os.path.join(PKG, "libpkvq_checked.so")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(ROOT, "include", "pkvq.h")]


def _stale(out: str) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in _deps())


def build(force: bool = False, bounds_check: bool = False, verbose: bool = False) -> str:
    out = LIB_CHECKED if bounds_check else LIB
    if not force and not _stale(out):
        return out
    objdir = os.path.join(PKG, "_build", "checked" if bounds_check else "release")
    os.makedirs(objdir, exist_ok=True)
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
                    "-I", os.path.join(ROOT, "include"), "-I", CSRC]
    if bounds_check:
        flags.append("-DPKVQ_BOUNDS_CHECK")
    if verbose:
        flags += ["-Xptxas", "-v"]
    def compile_one(src):
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        subprocess.run([NVCC] + flags + ["-c", src, "-o", obj], check=True)
        return obj

    # translation units compile independently (the tensor-core ones take
    # about a minute each)
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, _sources()))
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run([NVCC] + ARCH + ["-shared", "-o", tmp] + objs, check=True)
    os.replace(tmp, out)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--bounds-check", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true", help="print ptxas resource usage")
    a = ap.parse_args(argv)
    print(build(force=a.force, bounds_check=a.bounds_check, verbose=a.verbose))


if __name__ == "__main__":
    sys.exit(main())
