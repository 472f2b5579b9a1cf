"""Build ``libpagedkv.so`` in-tree with nvcc for sm_100a.

    python -m paged_kv_cache_364_b200.build [--force] [-j N]

Each source under ``csrc/`` compiles to an object in ``<repo>/_build/``; the
objects link into ``paged_kv_cache_364_b200/libpagedkv.so`` with the CUDA
runtime linked statically.  Rebuilds only what changed (sources or headers).
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libpagedkv.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _nvcc() -> str:
    exe = shutil.which("nvcc") or os.path.join(CUDA_HOME, "bin", "nvcc")
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libpagedkv.so")
    return exe


def _sources():
    out = []
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cpp")):
            out.append(os.path.join(CSRC, name))
    return out


def _headers():
    hs = [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    hs += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    return hs


def _compile_cmd(src: str, obj: str, extra: list[str]) -> list[str]:
    common = ["-O3", "-std=c++17", "-I", INCLUDE, "-I", CSRC, "-Xcompiler", "-fPIC"]
    if src.endswith(".cu"):
        return [_nvcc(), *ARCH, "-lineinfo", "--expt-relaxed-constexpr", *common, *extra,
                "-c", src, "-o", obj]
    return [_nvcc(), "-x", "c++", "-Wno-deprecated-gpu-targets", *common, *extra, "-c", src, "-o", obj]


def build(force: bool = False, jobs: int | None = None, verbose: bool = False,
          ptxas_info: bool = False) -> str:
    """Compile and link; returns the path of the shared library."""
    os.makedirs(BUILD, exist_ok=True)
    newest_header = max(os.path.getmtime(h) for h in _headers())
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    todo = []
    objs = []
    for src in _sources():
        obj = os.path.join(BUILD, os.path.basename(src) + ".o")
        objs.append(obj)
        stale = (not os.path.exists(obj) or os.path.getmtime(obj) < os.path.getmtime(src)
                 or os.path.getmtime(obj) < newest_header)
        if force or stale or ptxas_info:
            todo.append((src, obj))

    def run(job):
        src, obj = job
        cmd = _compile_cmd(src, obj, extra)
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"compiling {os.path.basename(src)} failed:\n{r.stdout}\n{r.stderr}")
        return src, r.stdout + r.stderr

    if todo:
        with ThreadPoolExecutor(max_workers=jobs or os.cpu_count() or 4) as ex:
            for src, log in ex.map(run, todo):
                if ptxas_info or verbose:
                    print(f"== {os.path.basename(src)}\n{log}", flush=True)
    if todo or not os.path.exists(LIB) or force:
        tmp = LIB + ".tmp"
        cmd = [_nvcc(), "-shared", *ARCH, "-o", tmp, *objs, "-cudart", "static", "-lpthread", "-ldl", "-lrt"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"linking libpagedkv.so failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
    return LIB


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-j", type=int, default=None)
    ap.add_argument("-v", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / spills / smem")
    a = ap.parse_args(argv)
    print(build(force=a.force, jobs=a.j, verbose=a.v, ptxas_info=a.ptxas_info))


if __name__ == "__main__":
    sys.exit(main())
