"""Builds libhstu.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: python -m hstu_sequential_transducer_b200.build [--force] [-j N] [--debug]
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libhstu.so")
# The debug build (-DHSTU_DEBUG): the attention kernels check the indices of
# their direct global accesses and report failures in the device status word
# (HSTU_DEVICE_BOUNDS) instead of making the access.  Loaded instead of the
# release library when HSTU_DEBUG_BUILD=1.
BUILD_DEBUG = os.path.join(ROOT, "_build_debug")
LIB_DEBUG = os.path.join(PKG, "libhstu_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                     "--expt-relaxed-constexpr", "-I" + INCLUDE, "-I" + CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def _mtime(p):
    return os.path.getmtime(p) if os.path.exists(p) else -1.0


def _flags(debug: bool):
    return NVCC_FLAGS + (["-DHSTU_DEBUG"] if debug else [])


def _compile(src: str, force: bool, debug: bool = False) -> str:
    obj = os.path.join(BUILD_DEBUG if debug else BUILD, os.path.basename(src)[:-3] + ".o")
    newest = max([_mtime(src)] + [_mtime(h) for h in _headers()])
    if force or _mtime(obj) < newest:
        cmd = [nvcc()] + _flags(debug) + ["-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    return obj


def source_hash(debug: bool = False) -> str:
    """Digest of every source, header and flag the library is built from."""
    h = hashlib.sha256(" ".join(_flags(debug)).encode())
    for p in _sources() + _headers():
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def build(force: bool = False, jobs: int = 0, debug: bool = False) -> str:
    """Compiles every csrc/*.cu and links libhstu.so (libhstu_debug.so with
    debug=True); returns its path.  Skips all work when the library was built
    from identical sources."""
    lib = LIB_DEBUG if debug else LIB
    stamp = lib + ".hash"
    digest = source_hash(debug)
    if not force and os.path.exists(lib) and os.path.exists(stamp) and \
            open(stamp).read().strip() == digest:
        return lib
    os.makedirs(BUILD_DEBUG if debug else BUILD, exist_ok=True)
    srcs = _sources()
    jobs = jobs or min(len(srcs), os.cpu_count() or 4)
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, debug), srcs))
    if force or _mtime(lib) < max(_mtime(o) for o in objs):
        cmd = [nvcc()] + ARCH + ["-shared", "-o", lib] + objs + ["-lcudart", "-ldl"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    with open(stamp, "w") as f:
        f.write(digest + "\n")
    return lib


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-j", type=int, default=0)
    ap.add_argument("--debug", action="store_true", help="build libhstu_debug.so (-DHSTU_DEBUG)")
    a = ap.parse_args(argv)
    print(build(a.force, a.j, a.debug))


if __name__ == "__main__":
    sys.exit(main())
