"""Build libkda.so in-tree from csrc/*.cu for sm_100a (B200).

    python -m decode_kda_chunked_b200.build [--verbose] [--jobs N] [--phase-profile]

Each translation unit is compiled with nvcc (-gencode arch=compute_100a,
code=sm_100a) into _build/, then linked into decode_kda_chunked_b200/libkda.so
with the CUDA runtime linked statically.  Only stale objects are rebuilt.

--phase-profile builds a separate diagnostic library, libkda_phase.so (objects in
_build/phase/), whose tensor-core prefill counts the cycles of each phase of its
chunk loop (see phase_profile.py); libkda.so itself never carries the counters.
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
PHASE_LIB = os.path.join(PKG, "libkda_phase.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
          "-Xptxas", "-warn-spills", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or install the CUDA toolkit")


def _deps(src: str):
    return [src] + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(out: str, deps) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str, verbose: bool, extra, build_dir: str = BUILD, force: bool = False) -> str:
    obj = os.path.join(build_dir, os.path.basename(src).replace(".cu", ".o"))
    if _stale(obj, _deps(src)) or force:
        cmd = [nvcc(), *ARCH, *CFLAGS, *extra, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return obj


def build(verbose: bool = False, jobs: int | None = None, extra=(), phase_profile: bool = False) -> str:
    """Build libkda.so (or, with ``phase_profile``, libkda_phase.so) and return its path.
    ``extra`` flags force a rebuild of every object."""
    build_dir = os.path.join(BUILD, "phase") if phase_profile else BUILD
    lib = PHASE_LIB if phase_profile else LIB
    flags = list(extra) + (["-DKDA_PHASE_PROFILE"] if phase_profile else [])
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    with cf.ThreadPoolExecutor(max_workers=jobs or min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, flags, build_dir, bool(extra)), srcs))
    if _stale(lib, objs) or extra:
        cmd = [nvcc(), *ARCH, "-shared", "-o", lib, *objs]
        subprocess.run(cmd, check=True)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--jobs", type=int, default=None)
    ap.add_argument("--phase-profile", action="store_true",
                    help="build the diagnostic libkda_phase.so with per-phase cycle counters")
    a = ap.parse_args()
    print(build(verbose=a.verbose, jobs=a.jobs, phase_profile=a.phase_profile))
    sys.exit(0)
