"""Build the CUDA library ``libsage_fp4.so`` in-tree for sm_100a with nvcc.

Each ``csrc/*.cu`` is compiled to an object under ``_build/`` and the objects are
linked into a shared library next to this file (CUDA runtime linked statically, so the
library loads on a machine without a GPU driver; the driver API is reached at run time
through cudaGetDriverEntryPoint). ``--checks`` builds the bounds-checked variant
``libsage_fp4_checks.so`` instead (compiled with SAGE_CHECKS: every computed global index
of the quantization and attention kernels is tested before the access; a failure is
reported in the device error word and the access skipped).

    python -m microscaling_fp4_quantized_b200.build [--force] [--verbose] [--checks]
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libsage_fp4.so")
LIB_CHECKS = os.path.join(PKG, "libsage_fp4_checks.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-v",
                 "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps():
    files = _sources()
    files += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    files += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return files + [os.path.abspath(__file__)]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _deps())


def build(force: bool = False, verbose: bool = False, checks: bool = False) -> str:
    lib = LIB_CHECKS if checks else LIB
    if not force and up_to_date(lib):
        return lib
    bdir = BUILD + ("_checks" if checks else "")
    os.makedirs(bdir, exist_ok=True)
    nvcc = _nvcc()
    flags = CFLAGS + (["-DSAGE_CHECKS"] if checks else [])

    def compile_one(src):
        obj = os.path.join(bdir, os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc] + flags + ["-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        return src, obj, r

    objs = []
    with cf.ThreadPoolExecutor(max_workers=4) as ex:
        for src, obj, r in ex.map(compile_one, _sources()):
            if r.returncode != 0:
                sys.stderr.write(r.stdout + r.stderr)
                raise RuntimeError(f"nvcc failed on {src}")
            if verbose:
                sys.stderr.write(r.stderr)
            objs.append(obj)
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc] + ARCH + ["-shared", "-o", tmp] + objs + ["-lrt", "-ldl", "-lpthread"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("link failed")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--checks", action="store_true", help="the bounds-checked variant")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, checks=a.checks))
