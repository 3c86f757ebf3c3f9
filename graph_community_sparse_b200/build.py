"""Compile libckv.so in-tree for sm_100a with nvcc (no GPU needed).

    python graph_community_sparse_b200/build.py [-v] [-f] [--debug | --all]

Objects go to graph_community_sparse_b200/_build/, the library to
graph_community_sparse_b200/libckv.so.  --debug builds libckv_debug.so
instead (objects in _build_debug/, compiled with CKV_DEBUG: every index a
caller's array feeds to a kernel is checked on the device, see
ckv_debug_build in include/ckv.h); --all builds both.  Only the ckv_* C
symbols are exported (linker version script); the CUDA runtime is linked
statically.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libckv.so")
BUILD_DEBUG = os.path.join(HERE, "_build_debug")
LIB_DEBUG = os.path.join(HERE, "libckv_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "-I", os.path.join(ROOT, "include"), "-I", CSRC]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _stale(out: str, deps) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, force: bool = False, debug: bool = False) -> str:
    nvcc = _nvcc()
    out_dir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug else (BUILD, LIB)
    flags = FLAGS + (["-DCKV_DEBUG"] if debug else [])
    os.makedirs(out_dir, exist_ok=True)
    headers = [os.path.join(ROOT, "include", "ckv.h")] + [
        os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")]
    objs = []
    jobs = []
    for src in sources():
        obj = os.path.join(out_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or _stale(obj, [src] + headers):
            cmd = [nvcc, *ARCH, *flags, "-c", src, "-o", obj]
            if verbose:
                cmd += ["-Xptxas", "-v"]
            jobs.append(cmd)

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, r

    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        for cmd, r in ex.map(run, jobs):
            if verbose or r.returncode:
                sys.stderr.write(r.stdout + r.stderr)
            if r.returncode:
                raise RuntimeError("nvcc failed: " + " ".join(cmd))
    if force or jobs or _stale(lib, objs):
        link = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", lib, *objs,
                "-Xlinker", "--version-script=" + os.path.join(CSRC, "ckv.map")]
        r = subprocess.run(link, capture_output=True, text=True)
        if r.returncode:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("link failed")
    return lib


if __name__ == "__main__":
    v, f = "-v" in sys.argv, "-f" in sys.argv
    if "--all" in sys.argv:
        print(build(v, f))
        print(build(v, f, debug=True))
    else:
        print(build(v, f, debug="--debug" in sys.argv))
