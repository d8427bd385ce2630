"""Builds libretnet.so (all CUDA sources of the package) for sm_100a in-tree.

    python -m linear_recurrent_sequence_02_b200.build [--force] [--verbose] [--debug]

Each csrc/*.cu is compiled to an object under _build/ (skipped when the
object is newer than its source and every header), then linked into
libretnet.so beside this file.  nvcc cross-compiles, so no GPU is needed.

`--debug` (build(variant="debug")) builds libretnet_debug.so from the same
sources with RETNET_CHECK_BOUNDS (index checks that report through the
device error word instead of trapping) and RETNET_TEST_HOOKS (the
retnet_test_set_hooks entry point that lets a test make a pipeline wait run
out); its objects go to _build/debug/.  The default library has neither.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libretnet.so")
DEBUG_LIB = os.path.join(PKG, "libretnet_debug.so")
VARIANTS = {
    "default": (BUILD, LIB, []),
    "debug": (os.path.join(BUILD, "debug"), DEBUG_LIB,
              ["-DRETNET_CHECK_BOUNDS", "-DRETNET_TEST_HOOKS"]),
}
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libretnet.so")
    return path


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(obj: str, src: str, headers) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(p) > t for p in [src, *headers, __file__])


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False,
          variant: str = "default") -> str:
    build_dir, lib_path, defines = VARIANTS[variant]
    os.makedirs(build_dir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = _headers()
    cc = nvcc()
    jobs = []
    for src in sources:
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        if force or _stale(obj, src, headers):
            cmd = [cc, *ARCH, *FLAGS, *defines, "-c", src, "-o", obj]
            if ptxas_verbose:
                cmd.insert(1, "-Xptxas=-v")
            jobs.append((src, cmd))

    def run(job):
        src, cmd = job
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        return src, r

    failed = []
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        for src, r in ex.map(run, jobs):
            if verbose or ptxas_verbose or r.returncode:
                sys.stderr.write(r.stdout + r.stderr)
            if r.returncode:
                failed.append(os.path.basename(src))
    if failed:
        raise RuntimeError(f"nvcc failed for: {', '.join(failed)}")

    objs = [os.path.join(build_dir, os.path.basename(s)[:-3] + ".o") for s in sources]
    if jobs or force or not os.path.exists(lib_path) or \
            any(os.path.getmtime(o) > os.path.getmtime(lib_path) for o in objs):
        tmp = lib_path + ".tmp"
        cmd = [cc, *ARCH, "-shared", "-o", tmp, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"linking {os.path.basename(lib_path)} failed")
        os.replace(tmp, lib_path)
    return lib_path


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    ap.add_argument("--debug", action="store_true",
                    help="build libretnet_debug.so (bounds checks and test hooks)")
    a = ap.parse_args()
    print(build(a.force, a.verbose, a.ptxas_verbose, "debug" if a.debug else "default"))


if __name__ == "__main__":
    main()
