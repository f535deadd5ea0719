"""Build libcvq.so in-tree with nvcc for sm_100a.

    python -m compressed_attention_cvq_b200.build          # build (incremental)
    python -m compressed_attention_cvq_b200.build --force  # rebuild everything
    python -m compressed_attention_cvq_b200.build --debug-bounds   # also the debug build

Each csrc/*.cu is compiled to an object under _build/ (skipped when the object is
newer than the source and the headers), then all objects are linked into
compressed_attention_cvq_b200/libcvq.so.  The debug build compiles the same sources with
-DCVQ_DEBUG_BOUNDS (device-side range checks that set CVQ_FAULT_BOUNDS in the fault word
and skip the access) into _build_debug/ and compressed_attention_cvq_b200/libcvq_debug.so,
which the binding loads when CVQ_LIBRARY=debug.
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
LIB = os.path.join(PKG, "libcvq.so")
BUILD_DEBUG = os.path.join(ROOT, "_build_debug")
LIB_DEBUG = os.path.join(PKG, "libcvq_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: libcvq cannot be built")


def _deps():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(obj: str, src: str) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(p) > t for p in [src, *_deps()])


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          debug_bounds: bool = False) -> str:
    build_dir, lib_path = (BUILD_DEBUG, LIB_DEBUG) if debug_bounds else (BUILD, LIB)
    extra = list(extra or []) + (["-DCVQ_DEBUG_BOUNDS"] if debug_bounds else [])
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    cc = nvcc()

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        if force or _stale(obj, src):
            cmd = [cc, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
            if verbose:
                print(" ".join(cmd), flush=True)
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
            if verbose and (r.stdout or r.stderr):
                print(r.stdout + r.stderr, flush=True)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, srcs))
    if (force or not os.path.exists(lib_path)
            or any(os.path.getmtime(o) > os.path.getmtime(lib_path) for o in objs)):
        cmd = [cc, *ARCH, "-shared", "-cudart", "static", "-o", lib_path, *objs, "-lpthread", "-ldl", "-lrt"]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib_path


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print register / smem usage")
    ap.add_argument("--debug-bounds", action="store_true",
                    help="also build libcvq_debug.so with device-side range checks")
    args = ap.parse_args(argv)
    extra = ["-Xptxas", "-v"] if args.ptxas_info else []
    lib = build(force=args.force or args.ptxas_info, verbose=args.verbose or args.ptxas_info, extra=extra)
    print(lib)
    if args.debug_bounds:
        print(build(force=args.force, verbose=args.verbose, debug_bounds=True))


if __name__ == "__main__":
    sys.exit(main())
