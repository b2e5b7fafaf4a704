"""Build libpagedattn.so in-tree with nvcc for sm_100a.

``python -m paged_kv_cache_359_b200.build [--force] [--ptxas-info]``

Each CUDA translation unit is compiled separately (in parallel) into
``_build/`` at the repository root, then linked with a static CUDA runtime
into ``paged_kv_cache_359_b200/libpagedattn.so``.  A unit is rebuilt when it
or any header is newer than its object.
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
LIB = os.path.join(PKG, "libpagedattn.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found")
    return path


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(obj, src, hdr_mtime):
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return os.path.getmtime(src) > t or hdr_mtime > t


def _compile(src, obj, ptxas_info):
    if src.endswith(".cu"):
        cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
               "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        if ptxas_info:
            cmd[1:1] = ["-Xptxas", "-v"]
    else:
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-I", INCLUDE, "-I", CSRC,
               "-I", "/usr/local/cuda/include", "-c", src, "-o", obj]
    res = subprocess.run(cmd, capture_output=True, text=True)
    return src, res.returncode, res.stdout + res.stderr


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          jobs: int | None = None) -> str:
    os.makedirs(BUILD, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))
    hdr_mtime = max((os.path.getmtime(h) for h in _headers()), default=0.0)
    build_py = os.path.getmtime(os.path.abspath(__file__))
    hdr_mtime = max(hdr_mtime, build_py)
    objs, todo = [], []
    for src in sources:
        obj = os.path.join(BUILD, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or ptxas_info or _stale(obj, src, hdr_mtime):
            todo.append((src, obj))
    jobs = jobs or max(1, min(len(todo), os.cpu_count() or 4))
    failed = []
    if todo:
        with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
            for src, rc, out in ex.map(lambda t: _compile(*t, ptxas_info), todo):
                if verbose or ptxas_info or rc != 0:
                    sys.stderr.write(f"== {os.path.basename(src)} (rc={rc})\n{out}")
                if rc != 0:
                    failed.append(src)
    if failed:
        raise RuntimeError("compilation failed: " + ", ".join(os.path.basename(f) for f in failed))
    lib_stale = force or not os.path.exists(LIB) or \
        any(os.path.getmtime(o) > os.path.getmtime(LIB) for o in objs)
    if lib_stale:
        tmp = LIB + ".tmp"
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("link failed:\n" + res.stdout + res.stderr)
        os.replace(tmp, LIB)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose, ptxas_info=args.ptxas_info))


if __name__ == "__main__":
    main()
