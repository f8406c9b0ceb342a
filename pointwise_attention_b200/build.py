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

SOURCES = ["hstu_api.cu", "fwd_sm100.cu", "bwd_sm100.cu", "plans.cu", "proj_sm100.cu", "cand_sm100.cu",
           "simt.cu", "selftest.cu", "noalloc.cu"]
HEADERS = ["internal.h", "ptx.cuh", "tile_math.cuh", "bounds.cuh"]
# The debug build: every data-derived index checked on the device (bounds.cuh).
BUILD_DEBUG = os.path.join(HERE, "_build_debug")
LIB_DEBUG = os.path.join(HERE, "libhstu_debug.so")


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


def build(force: bool = False, jobs: int = 4, verbose: bool = False,
          debug_bounds: bool = False) -> str:
    """Compiles the library (or, with debug_bounds, libhstu_debug.so with the
    device index checks of -DHSTU_DEBUG_BOUNDS); returns its path."""
    build_dir = BUILD_DEBUG if debug_bounds else BUILD
    lib = LIB_DEBUG if debug_bounds else LIB
    extra = ["-DHSTU_DEBUG_BOUNDS"] if debug_bounds else []
    os.makedirs(build_dir, exist_ok=True)
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "hstu.h")]
    objs, todo = [], []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(build_dir, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _stale(o, [s] + hdrs + [__file__]):
            todo.append((s, o))

    def compile_one(so):
        s, o = so
        cmd = [nvcc()] + cflags() + extra + ["-c", s, "-o", o]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (s, r.stdout, r.stderr))
        return s, r.stderr

    with cf.ThreadPoolExecutor(max_workers=max(1, jobs)) as ex:
        for s, log in ex.map(compile_one, todo):
            if verbose:
                print("== %s\n%s" % (os.path.basename(s), log))
            with open(os.path.join(build_dir, os.path.basename(s) + ".ptxas.txt"), "w") as f:
                f.write(log)
    if force or todo or _stale(lib, objs):
        tmp = lib + ".tmp%d" % os.getpid()
        cmd = [nvcc(), "-shared", "-cudart", "static", "-o", tmp] + objs + [
            "-Xlinker", "--exclude-libs,ALL", "-lrt", "-ldl", "-lpthread"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n%s\n%s" % (r.stdout, r.stderr))
        os.replace(tmp, lib)
    return lib


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=4)
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true",
                    help="build libhstu_debug.so with device-side index checks")
    args = ap.parse_args(argv)
    print(build(args.force, args.jobs, args.verbose, args.debug_bounds))


if __name__ == "__main__":
    sys.exit(main())
