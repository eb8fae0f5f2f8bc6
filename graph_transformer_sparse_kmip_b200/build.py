"""Build libkmip.so (CUDA, sm_100a) in-tree with nvcc.

    python -m graph_transformer_sparse_kmip_b200.build [--force] [--jobs N]

Each ``csrc/*.cu`` compiles to an object under ``_build/`` (skipped when the
object is newer than every source and header), then all objects link into
``graph_transformer_sparse_kmip_b200/libkmip.so`` with the CUDA runtime
linked statically, so the library needs only the driver at run time.

``--debug-bounds`` builds ``libkmip_debug.so`` instead (objects under
``_build/debug/``) with KMIP_DEBUG_BOUNDS defined: the kernels then check
every key index they are about to read against the query's graph and record
KMIP_ERR_BAD_INDEX in the status word instead of reading out of range.  The
binding loads it when KMIP_DEBUG_BOUNDS=1.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libkmip.so")
LIB_DEBUG = os.path.join(PKG, "libkmip_debug.so")
NVCC = os.environ.get("NVCC", "nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                  + glob.glob(os.path.join(ROOT, "include", "*.h")))


def _compile(src: str, force: bool, verbose: bool, debug: bool = False) -> str:
    obj = os.path.join(BUILD, "debug" if debug else "", os.path.basename(src)[:-3] + ".o")
    newest = max(os.path.getmtime(p) for p in [src] + _headers())
    if not force and os.path.exists(obj) and os.path.getmtime(obj) >= newest:
        return obj
    cmd = [NVCC, *ARCH, *FLAGS, *(["-DKMIP_DEBUG_BOUNDS"] if debug else []), "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose:
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, jobs: int | None = None, verbose: bool = False,
          debug_bounds: bool = False) -> str:
    os.makedirs(os.path.join(BUILD, "debug") if debug_bounds else BUILD, exist_ok=True)
    lib = LIB_DEBUG if debug_bounds else LIB
    srcs = _sources()
    with cf.ThreadPoolExecutor(max_workers=jobs or min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, verbose, debug_bounds), srcs))
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs):
        cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", lib, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=None)
    ap.add_argument("-v", "--verbose", action="store_true", help="print ptxas resource usage")
    ap.add_argument("--debug-bounds", action="store_true",
                    help="build libkmip_debug.so with device-side index checks")
    args = ap.parse_args()
    print(build(force=args.force, jobs=args.jobs, verbose=args.verbose,
                debug_bounds=args.debug_bounds))
