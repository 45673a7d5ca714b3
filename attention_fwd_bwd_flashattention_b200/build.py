"""Build the CUDA library in-tree: csrc/*.cu -> _lib/librelpos_attn.so (sm_100a).

Run ``python -m attention_fwd_bwd_flashattention_b200.build``; nvcc cross-compiles
without a GPU.  The shared library exports exactly the C ABI of include/relpos_attn.h.
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.join(PKG, "_lib")
LIBNAME = "librelpos_attn.so"
DEBUG_LIBNAME = "librelpos_attn_debug.so"  # RELPOS_DEBUG: index checks of the kernels' stores
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def lib_path(debug: bool = False) -> str:
    return os.path.join(LIBDIR, DEBUG_LIBNAME if debug else LIBNAME)


def up_to_date(debug: bool = False) -> bool:
    out = lib_path(debug)
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + [os.path.join(INCLUDE, "relpos_attn.h")]
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force: bool = False, verbose: bool = False, extra=None, debug: bool = False) -> str:
    """Compile (if stale) and return the path of the shared library (debug: the
    RELPOS_DEBUG build, whose kernels check the indices of their stores).  Each source is
    compiled by its own nvcc process (in parallel), then the objects are linked."""
    if not force and up_to_date(debug):
        return lib_path(debug)
    os.makedirs(LIBDIR, exist_ok=True)
    objdir = os.path.join(LIBDIR, "obj_debug" if debug else "obj")
    os.makedirs(objdir, exist_ok=True)
    flags = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden", "--expt-relaxed-constexpr",
             "-I", INCLUDE, "-I", CSRC, *(["-DRELPOS_DEBUG"] if debug else []), *(extra or [])]

    def compile_one(src):
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc(), *flags, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        r = subprocess.run(cmd, capture_output=True, text=True)
        return src, obj, r

    with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, min(len(sources()), os.cpu_count() or 1))) as ex:
        results = list(ex.map(compile_one, sources()))
    failed = False
    for src, _, r in results:
        if r.stdout or r.stderr:
            print(r.stdout + r.stderr, file=sys.stderr, end="")
        if r.returncode != 0:
            print(f"nvcc failed: {src}", file=sys.stderr)
            failed = True
    if failed:
        raise subprocess.CalledProcessError(1, "nvcc")
    tmp = lib_path(debug) + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *[o for _, o, _ in results]]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib_path(debug))
    return lib_path(debug)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, extra=["-Xptxas", "-v"] if "--ptxas" in sys.argv else None,
                debug="--debug" in sys.argv))
