"""Build librlt.so (sm_100a) in-tree with nvcc.

    python stateful_decoding_b200/build.py [--force] [--jobs N] [--ptxas-v] [--debug]

(Run it by path, or load it with ``load_builder()``: importing the package
itself loads the library it builds.)

Each .cu under csrc/ compiles to an object in _build/ (in parallel), then
they link into stateful_decoding_b200/librlt.so.  Objects are rebuilt when
their source or any header changed.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "librlt.so")
# the bounds-checking variant (RLT_DEBUG=1): same sources, own objects
DEBUG_BUILD = os.path.join(BUILD, "debug")
DEBUG_LIB = os.path.join(HERE, "librlt_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-Xcompiler", "-Wall", "-I", os.path.join(ROOT, "include"), "-I", CSRC]


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _headers():
    return [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + \
        [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))]


def _compile(src: str, force: bool, extra, outdir: str = BUILD) -> str:
    obj = os.path.join(outdir, os.path.basename(src)[:-3] + ".o")
    newest = max([os.path.getmtime(src)] + [os.path.getmtime(h) for h in _headers()])
    if not force and os.path.exists(obj) and os.path.getmtime(obj) >= newest:
        return obj
    cmd = [NVCC] + ARCH + FLAGS + list(extra) + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if r.stderr.strip():
        sys.stderr.write(r.stderr)
    return obj


def load_builder():
    """This module, loaded by file path without importing the package."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("rlt_build", os.path.abspath(__file__))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def build(force: bool = False, jobs: int | None = None, extra=(), debug: bool = False) -> str:
    """Build librlt.so, or with debug=True librlt_debug.so (RLT_DEBUG=1: the
    kernels' bounds checks compiled in)."""
    outdir, lib = (DEBUG_BUILD, DEBUG_LIB) if debug else (BUILD, LIB)
    extra = list(extra) + (["-DRLT_DEBUG=1"] if debug else [])
    os.makedirs(outdir, exist_ok=True)
    srcs = _sources()
    jobs = jobs or min(8, os.cpu_count() or 4)
    with cf.ThreadPoolExecutor(jobs) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, extra, outdir), srcs))
    if not force and os.path.exists(lib) and \
            os.path.getmtime(lib) >= max(os.path.getmtime(o) for o in objs):
        return lib
    cmd = [NVCC] + ARCH + ["-shared", "-o", lib] + objs + ["-lcudart", "-lcuda"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=None)
    ap.add_argument("--ptxas-v", action="store_true", help="print register/smem usage")
    ap.add_argument("--debug", action="store_true",
                    help="build librlt_debug.so (RLT_DEBUG=1 bounds checks)")
    a = ap.parse_args()
    extra = ["-Xptxas", "-v"] if a.ptxas_v else []
    print(build(force=a.force or a.ptxas_v, jobs=a.jobs, extra=extra, debug=a.debug))
