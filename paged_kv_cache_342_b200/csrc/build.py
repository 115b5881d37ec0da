"""Build libpa.so (the C-ABI library) in-tree for B200 (sm_100a).

    python paged_kv_cache_342_b200/csrc/build.py [--verbose-ptxas] [--jobs N] [--force]

(A plain script beside the sources: it must run before the package, which refuses
to import without the library, can be imported.)

Each source compiles to an object under ``_build/`` in parallel; the objects link
into ``paged_kv_cache_342_b200/libpa.so`` with the CUDA runtime linked statically.
A source is recompiled only when it, or a header, is newer than its object.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

CSRC = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(CSRC)
ROOT = os.path.dirname(PKG)
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libpa.so")
HEADERS = [os.path.join(ROOT, "include", "pa.h")] + [
    os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
              "--expt-relaxed-constexpr", f"-I{os.path.join(ROOT, 'include')}"] + ARCH


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cpp")))


def _stale(src: str, obj: str) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return os.path.getmtime(src) > t or any(os.path.getmtime(h) > t for h in HEADERS)


def build(verbose_ptxas: bool = False, jobs: int | None = None, force: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    cc = nvcc()
    objs, todo = [], []
    for src in sources():
        obj = os.path.join(BUILD, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or _stale(src, obj):
            flags = list(NVCC_FLAGS)
            if verbose_ptxas and src.endswith(".cu"):
                flags += ["-Xptxas", "-v"]
            todo.append([cc, *flags, "-c", src, "-o", obj])

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, r

    failed = []
    with ThreadPoolExecutor(jobs or max(1, min(8, os.cpu_count() or 1))) as ex:
        for cmd, r in ex.map(run, todo):
            if verbose_ptxas or r.returncode:
                sys.stderr.write(r.stdout + r.stderr)
            if r.returncode:
                failed.append(cmd[-3])
    if failed:
        raise RuntimeError(f"nvcc failed for {failed}")
    if todo or not os.path.exists(LIB):
        link = [cc, "-shared", *ARCH, "-o", LIB + ".tmp", *objs, "-cudart", "static"]
        r = subprocess.run(link, capture_output=True, text=True)
        if r.returncode:
            raise RuntimeError("link failed:\n" + r.stdout + r.stderr)
        os.replace(LIB + ".tmp", LIB)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--jobs", type=int, default=None)
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(a.verbose_ptxas, a.jobs, a.force))


if __name__ == "__main__":
    main()
