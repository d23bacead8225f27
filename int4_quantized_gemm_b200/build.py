"""Build libqg.so (the CUDA library behind include/qg.h) in-tree with nvcc.

    python int4_quantized_gemm_b200/build.py [--force] [--jobs N] [--debug]

--debug builds libqg_debug.so instead: the same sources with QG_DEBUG defined,
whose kernels check TMA coordinates and shared/tensor memory offsets on the
device and report a failed check through the status word (qg_debug_checks()).

Compiles every csrc/*.cu for sm_100a only (-gencode arch=compute_100a,code=sm_100a)
into int4_quantized_gemm_b200/_build/*.o and links int4_quantized_gemm_b200/libqg.so
against the static CUDA runtime (no link-time libcuda dependency: the driver's
cuTensorMapEncodeTiled is fetched at run time).  Objects are rebuilt when their
source or any csrc header / include/qg.h is newer.  Cross-compiles without a GPU.
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
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libqg.so")
BUILD_DEBUG = os.path.join(PKG, "_build_debug")
LIB_DEBUG = os.path.join(PKG, "libqg_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2,-Wall",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libqg.so")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(ROOT, "include", "qg.h")]


def _stale(obj: str, deps: list[str]) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str, obj: str, verbose_ptxas: bool, debug: bool = False) -> str:
    cmd = [nvcc(), *NVCC_FLAGS, *(["-DQG_DEBUG"] if debug else []), "-c", src, "-o", obj + ".tmp"]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
    os.replace(obj + ".tmp", obj)
    return r.stderr


def build(force: bool = False, jobs: int | None = None, verbose_ptxas: bool = False, debug: bool = False) -> str:
    BUILD, LIB = (BUILD_DEBUG, LIB_DEBUG) if debug else (globals()["BUILD"], globals()["LIB"])
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    heads = _headers()
    todo = []
    objs = []
    for src in srcs:
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or _stale(obj, [src, *heads]):
            todo.append((src, obj))
    if todo:
        with cf.ThreadPoolExecutor(max_workers=jobs or min(8, len(todo))) as ex:
            for log in ex.map(lambda so: _compile(*so, verbose_ptxas, debug), todo):
                if verbose_ptxas and log:
                    sys.stderr.write(log)
    if todo or not os.path.exists(LIB) or _stale(LIB, objs):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "--cudart", "static",
               "-o", tmp, *objs, "-ldl", "-lpthread", "-lrt"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
    return LIB


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=None)
    ap.add_argument("--ptxas-verbose", action="store_true", help="print register/shared-memory use")
    ap.add_argument("--debug", action="store_true", help="build libqg_debug.so (device-side checks)")
    a = ap.parse_args()
    print(build(force=a.force, jobs=a.jobs, verbose_ptxas=a.ptxas_verbose, debug=a.debug))


if __name__ == "__main__":
    main()
