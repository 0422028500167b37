"""Build the CUDA library in-tree: exact_attention_115_b200/libfa_b200.so.

Compiles every ``csrc/*.cu`` for sm_100a with nvcc (in parallel), then links
one shared library exporting the C ABI declared in ``include/fa.h``.  Run as
``python -m exact_attention_115_b200.build`` (``--verbose`` shows ptxas
register/spill reports; ``--debug`` builds libfa_b200_debug.so, the same
library with FA_DEBUG index checks in every kernel, reported by fa_status as
FA_ERR_BOUNDS).  No GPU is needed to build.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libfa_b200.so")
DEBUG_LIB = os.path.join(PKG, "libfa_b200_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _compile(src: str, verbose: bool, debug: bool = False) -> tuple[str, str]:
    out_dir = os.path.join(BUILD, "debug") if debug else BUILD
    obj = os.path.join(out_dir, os.path.basename(src) + ".o")
    cmd = [nvcc(), *ARCH, *FLAGS, *(["-DFA_DEBUG"] if debug else []), "-c", src, "-o", obj]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC)
                        if f.endswith((".cuh", ".h"))] + [os.path.join(INCLUDE, "fa.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(verbose: bool = False, force: bool = False, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    if not force and not _stale(lib):
        return lib
    os.makedirs(os.path.join(BUILD, "debug") if debug else BUILD, exist_ok=True)
    srcs = sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(lambda s: _compile(s, verbose, debug), srcs))
    if verbose:
        for (obj, log), src in zip(results, srcs):
            print(f"== {os.path.basename(src)}\n{log}", file=sys.stderr)
    objs = [o for o, _ in results]
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--debug", action="store_true")
    a = ap.parse_args()
    print(build(verbose=a.verbose, force=a.force, debug=a.debug))
