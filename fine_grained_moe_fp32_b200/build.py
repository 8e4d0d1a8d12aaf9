"""Build libmoe_b200.so (the C-ABI CUDA library) in-tree for sm_100a.

    python -m fine_grained_moe_fp32_b200.build [--force] [--verbose] [--checks]

Each csrc/*.cu is compiled to an object under _build/ (in parallel), then the
objects are linked into fine_grained_moe_fp32_b200/libmoe_b200.so with the
CUDA runtime linked statically.  --checks builds the same sources with
-DMOE_CHECKS=1 (device bounds checks that record MOE_ERR_BOUNDS, a guard
zone after every workspace region) into libmoe_b200_checks.so, objects
under _build/checks/.
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
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmoe_b200.so")
LIB_CHECKS = os.path.join(PKG, "libmoe_b200_checks.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
         "-Xcompiler", "-fPIC,-O3", f"-I{INCLUDE}", f"-I{CSRC}"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, checks: bool = False) -> str:
    """Compile and link the library (the MOE_CHECKS variant when ``checks``)
    unless it is newer than every source."""
    lib = LIB_CHECKS if checks else LIB
    if not force and up_to_date(lib):
        return lib
    bdir = os.path.join(BUILD, "checks") if checks else BUILD
    os.makedirs(bdir, exist_ok=True)
    nvcc = _nvcc()
    flags = FLAGS + (["-DMOE_CHECKS=1"] if checks else [])

    def compile_one(src):
        obj = os.path.join(bdir, os.path.basename(src).replace(".cu", ".o"))
        cmd = [nvcc, *ARCH, *flags, "-c", src, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stdout + r.stderr

    with cf.ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        results = list(ex.map(compile_one, _sources()))
    if verbose:
        for _, log in results:
            if log.strip():
                print(log, file=sys.stderr)
    objs = [o for o, _ in results]
    tmp = lib + ".tmp"
    cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--checks", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, checks=a.checks))


if __name__ == "__main__":
    main()
