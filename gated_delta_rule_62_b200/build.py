"""Build libkda.so in-tree with nvcc for sm_100a (B200).

    python -m gated_delta_rule_62_b200.build [--force] [--verbose] [--debug] [--nvtx] [--tc-inverse]

Each ``csrc/*.cu`` is compiled to an object under ``_build/`` (in parallel) and
linked with the static CUDA runtime into ``gated_delta_rule_62_b200/libkda.so``.
Works without a GPU (nvcc cross-compiles).

``--debug`` builds ``libkda_debug.so`` instead, with -DKDA_DEBUG: every global
access at a computed address is checked against its buffer's byte range, and an
access outside it is skipped and reported through the device status word
(KDA_ERR_INTERNAL). ``--nvtx`` adds an NVTX range per library call (-DKDA_NVTX).
``--tc-inverse`` builds ``libkda_tcinv.so``, whose split-role prefill inverts the 64x64 unit
lower-triangular matrix with three rounds of tcgen05 MMAs (-DKDA_TC_INVERSE) instead of the
warp-level tf32 merges; it is correct and slower, and kept for that comparison.
Load another build than ``libkda.so`` by setting KDA_LIB to its path.
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
LIB = os.path.join(PKG, "libkda.so")
DEBUG_LIB = os.path.join(PKG, "libkda_debug.so")
TCINV_LIB = os.path.join(PKG, "libkda_tcinv.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False, debug: bool = False,
          nvtx: bool = False, tc_inverse: bool = False) -> str:
    lib = DEBUG_LIB if debug else (TCINV_LIB if tc_inverse else LIB)
    if not force and not nvtx and up_to_date(lib):
        return lib
    objdir = os.path.join(BUILD, "debug" if debug else ("tcinv" if tc_inverse else ("nvtx" if nvtx else "release")))
    os.makedirs(objdir, exist_ok=True)
    cc = nvcc()
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    if debug:
        extra += ["-DKDA_DEBUG"]
    if nvtx:
        extra += ["-DKDA_NVTX"]
    if tc_inverse:
        extra += ["-DKDA_TC_INVERSE"]

    def compile_one(src):
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [cc, *ARCH, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stderr}")
        if verbose or ptxas_info:
            sys.stderr.write(r.stderr)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, _sources()))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [cc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs, "-lrt", "-ldl", "-lpthread"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    ap.add_argument("--debug", action="store_true")
    ap.add_argument("--nvtx", action="store_true")
    ap.add_argument("--tc-inverse", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_info=a.ptxas_info, debug=a.debug, nvtx=a.nvtx,
                tc_inverse=a.tc_inverse))
