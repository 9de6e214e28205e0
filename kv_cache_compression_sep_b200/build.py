"""Builds libsepattn.so (the sm_100a kernels + C ABI) in the package directory with nvcc.

Usage: python -m kv_cache_compression_sep_b200.build [--force] [--jobs N]
Each translation unit is compiled to an object in _build/ and linked into one shared library
(static CUDA runtime, driver entry points resolved at run time, no libcuda link).
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
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsepattn.so")
SOURCES = ["k_mask.cu", "k_attn_fwd.cu", "k_attn_bwd.cu", "k_sepcache.cu", "k_scratch.cu", "api.cpp"]
HEADERS = ["sep_common.cuh", "sep_tiles.cuh", "sep_launch.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I" + os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libsepattn.so")


def _mtime(p):
    return os.path.getmtime(p) if os.path.exists(p) else -1.0


def _deps_mtime():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "sepattn.h"))
    return max(_mtime(f) for f in files)


def up_to_date() -> bool:
    return _mtime(LIB) >= _deps_mtime()


def _compile(src: str) -> str:
    os.makedirs(BUILD, exist_ok=True)
    obj = os.path.join(BUILD, src + ".o")
    if _mtime(obj) >= _deps_mtime():
        return obj
    cmd = [nvcc(), *ARCH, *FLAGS, "-c", os.path.join(CSRC, src), "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    return obj


def build(force: bool = False, jobs: int = 0) -> str:
    if not force and up_to_date():
        return LIB
    if force and os.path.isdir(BUILD):
        shutil.rmtree(BUILD)
    jobs = jobs or min(len(SOURCES), os.cpu_count() or 1)
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        objs = list(ex.map(_compile, SOURCES))
    tmp = LIB + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=0)
    args = ap.parse_args()
    print(build(force=args.force, jobs=args.jobs))
    sys.exit(0)
