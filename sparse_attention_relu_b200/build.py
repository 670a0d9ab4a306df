"""Builds libdsa.so in-tree from csrc/*.cu for sm_100a (nvcc, no JIT cache).

    python -m sparse_attention_relu_b200.build [--force] [--trace]

--trace also builds libdsa_trace.so, a diagnostic copy whose attention kernel
records per-tile clock64 stamps (attn_tc.cu compiled with -DDSA_ATTN_TRACE;
stage_bench.py --trace reads them).  The product path never loads it.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libdsa.so")
TRACE_LIB = os.path.join(HERE, "libdsa_trace.so")
OBJ_DIR = os.path.join(HERE, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-I" + os.path.join(ROOT, "include")]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [
        os.path.join(ROOT, "include", "dsa.h")]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _deps())


def _compile(src: str, extra=(), obj_dir: str = OBJ_DIR) -> str:
    obj = os.path.join(obj_dir, os.path.basename(src) + ".o")
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    return obj


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    srcs = _sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(_compile, srcs))
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    if verbose:
        print("built", LIB)
    return LIB


def build_trace(verbose: bool = False) -> str:
    """libdsa.so's objects with attn_tc.cu recompiled under -DDSA_ATTN_TRACE."""
    if os.path.exists(TRACE_LIB) and up_to_date() and all(
            os.path.getmtime(p) <= os.path.getmtime(TRACE_LIB) for p in _deps()):
        return TRACE_LIB
    attn = os.path.join(CSRC, "attn_tc.cu")
    others = [os.path.join(OBJ_DIR, os.path.basename(s) + ".o") for s in _sources() if s != attn]
    build(force=not all(os.path.exists(o) for o in others))
    tdir = os.path.join(OBJ_DIR, "trace")
    os.makedirs(tdir, exist_ok=True)
    objs = [_compile(attn, ["-DDSA_ATTN_TRACE"], tdir)] + others
    tmp = TRACE_LIB + f".tmp{os.getpid()}"
    r = subprocess.run([NVCC, *ARCH, "-shared", "-o", tmp, *objs], capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, TRACE_LIB)
    if verbose:
        print("built", TRACE_LIB)
    return TRACE_LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    if "--trace" in sys.argv:
        build_trace(verbose=True)
