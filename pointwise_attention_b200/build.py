"""Builds libhstu.so (sm_100a) in-tree with nvcc.

    python -m pointwise_attention_b200.build [--force] [--jobs N]

Each source under csrc/ is compiled for ``-gencode arch=compute_100a,code=sm_100a``
with ``-lineinfo``; the shared library links the CUDA runtime statically and
takes ``cuTensorMapEncodeTiled`` from the driver at run time, so it loads on a
machine without a GPU (the CPU tests check its exported symbols there).
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libhstu.so")

SOURCES = ["hstu_api.cu", "fwd_sm100.cu", "bwd_sm100.cu", "proj_sm100.cu", "cand_sm100.cu",
           "simt.cu", "selftest.cu", "noalloc.cu"]
HEADERS = ["internal.h", "ptx.cuh", "tile_math.cuh"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libhstu")


def cflags():
    return ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
            "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE,
            "-I", CSRC, "--expt-relaxed-constexpr", "-Xptxas", "-v"]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, jobs: int = 4, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "hstu.h")]
    objs, todo = [], []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _stale(o, [s] + hdrs + [__file__]):
            todo.append((s, o))

    def compile_one(so):
        s, o = so
        cmd = [nvcc()] + cflags() + ["-c", s, "-o", o]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (s, r.stdout, r.stderr))
        return s, r.stderr

    with cf.ThreadPoolExecutor(max_workers=max(1, jobs)) as ex:
        for s, log in ex.map(compile_one, todo):
            if verbose:
                print("== %s\n%s" % (os.path.basename(s), log))
            with open(os.path.join(BUILD, os.path.basename(s) + ".ptxas.txt"), "w") as f:
                f.write(log)
    if force or todo or _stale(LIB, objs):
        tmp = LIB + ".tmp%d" % os.getpid()
        cmd = [nvcc(), "-shared", "-cudart", "static", "-o", tmp] + objs + [
            "-Xlinker", "--exclude-libs,ALL", "-lrt", "-ldl", "-lpthread"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n%s\n%s" % (r.stdout, r.stderr))
        os.replace(tmp, LIB)
    return LIB


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=4)
    ap.add_argument("-v", "--verbose", action="store_true")
    args = ap.parse_args(argv)
    print(build(args.force, args.jobs, args.verbose))


if __name__ == "__main__":
    sys.exit(main())
