"""Build the CUDA library libq4.so (sm_100a only) in-tree with nvcc, and its debug build libq4_debug.so
(Q4_DEBUG: every global index a kernel computes is checked against its buffer, a failed check is
reported as Q4_ERR_BOUNDS instead of being made).

Usage: python -m moe_linear_layers_b200.build_lib [--force] [--jobs N] [--debug]
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
OUT = os.path.join(HERE, "libq4.so")
BUILD = os.path.join(ROOT, "_build")
OUT_DEBUG = os.path.join(HERE, "libq4_debug.so")
BUILD_DEBUG = os.path.join(ROOT, "_build", "debug")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h")))


def _stale(obj, src, hdr_mtime):
    return not os.path.exists(obj) or os.path.getmtime(obj) < max(os.path.getmtime(src), hdr_mtime)


def build(force: bool = False, jobs: int = 0, verbose: bool = False, extra: list | None = None,
          debug: bool = False) -> str:
    build_dir, out = (BUILD_DEBUG, OUT_DEBUG) if debug else (BUILD, OUT)
    extra = (extra or []) + (["-DQ4_DEBUG"] if debug else [])
    os.makedirs(build_dir, exist_ok=True)
    hdr_mtime = max([os.path.getmtime(h) for h in headers()] + [os.path.getmtime(__file__)])
    srcs = sources()
    objs = [os.path.join(build_dir, os.path.basename(s) + ".o") for s in srcs]
    todo = [(s, o) for s, o in zip(srcs, objs) if force or _stale(o, s, hdr_mtime)]

    def compile_one(so):
        s, o = so
        cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", s, "-o", o]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {os.path.basename(s)}:\n{r.stdout}\n{r.stderr}")
        return r.stderr

    if todo:
        with cf.ThreadPoolExecutor(max_workers=jobs or min(8, os.cpu_count() or 1)) as ex:
            for msg in ex.map(compile_one, todo):
                if verbose and msg:
                    print(msg)
    if todo or not os.path.exists(out):
        tmp = out + f".tmp{os.getpid()}"
        cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static", "-ldl"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, out)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=0)
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print register/spill usage")
    ap.add_argument("--debug", action="store_true", help="build libq4_debug.so (Q4_DEBUG bounds checks)")
    a = ap.parse_args()
    print(build(force=a.force, jobs=a.jobs, verbose=a.verbose or a.ptxas_v,
                extra=["-Xptxas", "-v"] if a.ptxas_v else None, debug=a.debug))
