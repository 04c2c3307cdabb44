"""Builds libqsa.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m sparse_attention_decode_02_b200.build [--force] [--verbose] [--checked]

Each translation unit under csrc/ is compiled in parallel into _build/, then linked
into sparse_attention_decode_02_b200/libqsa.so. The build is skipped when the library
is newer than every source and header.

--checked builds libqsa_checked.so instead (objects in _build_checked/), compiled with
-DQSA_CHECKED: bounds guards on the kernels' data-dependent writes record
QSA_ERR_BAD_INDEX in the layer status and skip the access (a stand-in for a memory
sanitizer). Point the binding at it with QSA_LIBRARY=<path to libqsa_checked.so>.

--timeline builds libqsa_timeline.so (objects in _build_timeline/), compiled with
-DQSA_TIMELINE: the decode-step kernels record %globaltimer marks for one chosen layer
(csrc/qsa_timeline.cuh), read back through qsa_tl_arm_<kernel> / qsa_tl_read_<kernel>.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libqsa.so")
LIB_CHECKED = os.path.join(PKG, "libqsa_checked.so")
LIB_TIMELINE = os.path.join(PKG, "libqsa_timeline.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "--expt-relaxed-constexpr", "-diag-suppress", "177"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or put CUDA's bin directory on PATH")


def _inputs():
    return (sorted(glob.glob(os.path.join(CSRC, "*.cu"))),
            sorted(glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                   + glob.glob(os.path.join(ROOT, "include", "*.h"))))


def up_to_date(lib: str = LIB) -> bool:
    srcs, hdrs = _inputs()
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in srcs + hdrs + [__file__])


def build(force: bool = False, verbose: bool = False, checked: bool = False, timeline: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB_TIMELINE if timeline else LIB
    if not force and up_to_date(lib):
        return lib
    nvcc = _nvcc()
    srcs, _ = _inputs()
    build_dir = BUILD + ("_checked" if checked else "_timeline" if timeline else "")
    os.makedirs(build_dir, exist_ok=True)
    extra = (["-DQSA_CHECKED"] if checked else []) + (["-DQSA_TIMELINE"] if timeline else [])

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc, *ARCH, *FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-c", src, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stderr}")
        if verbose and r.stderr:
            sys.stderr.write(r.stderr)
        return obj

    with cf.ThreadPoolExecutor(max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(compile_one, srcs))
    tmp = lib + ".tmp"
    r = subprocess.run([nvcc, *ARCH, "-shared", "-o", tmp, *objs], capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, checked="--checked" in sys.argv,
                timeline="--timeline" in sys.argv))
