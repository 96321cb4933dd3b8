"""Build the sm_100a shared library in-tree: block_sparse_masked_x128_b200/_lib/libfa_b200.so.

    python block_sparse_masked_x128_b200/build.py [--verbose] [--ptxas-info] [--force] [--debug]

(Run it as a file, not as a package module: importing the package loads the library.)

Each .cu file is compiled to an object in parallel (nvcc cross-compiles for sm_100a without
a GPU), then linked into one shared library exporting the C ABI of include/fa_b200.h.
Objects are rebuilt only when a source or header is newer.  `--ptxas-info` prints the
registers and shared memory of every kernel (nvcc -Xptxas -v).
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
LIBDIR = os.path.join(PKG, "_lib")
LIB = os.path.join(LIBDIR, "libfa_b200.so")
TRACE_LIB = os.path.join(LIBDIR, "libfa_b200_trace.so")
DEBUG_LIB = os.path.join(LIBDIR, "libfa_b200_debug.so")
SOURCES = ["api.cu", "mask_builder.cu", "attn_fwd.cu", "noalloc.cu", "masked_softmax.cu", "attn_bwd.cu", "decode.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _flags(ptxas_info: bool, trace: bool = False, debug: bool = False) -> list:
    f = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                "-I", INCLUDE, "-I", CSRC, "--expt-relaxed-constexpr"]
    if ptxas_info:
        f += ["-Xptxas", "-v"]
    if trace:
        f += ["-DFA_TRACE"]
    if debug:
        f += ["-DFA_DEBUG"]
    return f


def _headers() -> list:
    hs = [os.path.join(CSRC, h) for h in os.listdir(CSRC) if h.endswith((".h", ".cuh"))]
    return hs + [os.path.join(INCLUDE, h) for h in os.listdir(INCLUDE) if h.endswith(".h")]


def _compile(src: str, flags: list, force: bool, build_dir: str = BUILD) -> tuple:
    obj = os.path.join(build_dir, os.path.splitext(src)[0] + ".o")
    srcp = os.path.join(CSRC, src)
    newest = max(os.path.getmtime(p) for p in [srcp] + _headers())
    if not force and os.path.exists(obj) and os.path.getmtime(obj) >= newest:
        return obj, ""
    cmd = [_nvcc()] + flags + ["-c", srcp, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    return obj, r.stdout + r.stderr


def build(verbose: bool = False, ptxas_info: bool = False, force: bool = False,
          trace: bool = False, debug: bool = False) -> str:
    """Build the library; trace=True builds the phase-tracing variant, debug=True the variant
    whose kernels check metadata indices (FA_DEBUG), each under its own name."""
    variant = "trace" if trace else ("debug" if debug else "")
    build_dir = os.path.join(BUILD, variant) if variant else BUILD
    lib = TRACE_LIB if trace else (DEBUG_LIB if debug else LIB)
    os.makedirs(build_dir, exist_ok=True)
    os.makedirs(LIBDIR, exist_ok=True)
    flags = _flags(ptxas_info, trace, debug)
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(lambda s: _compile(s, flags, force or ptxas_info, build_dir), SOURCES))
    objs = [o for o, _ in results]
    if verbose or ptxas_info:
        for _, log in results:
            if log:
                print(log)
    newest_obj = max(os.path.getmtime(o) for o in objs)
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < newest_obj:
        cmd = [_nvcc()] + ARCH + ["-shared", "-o", lib] + objs + ["-lcudart_static", "-ldl", "-lrt", "-lpthread"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    return lib


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--trace", action="store_true", help="build the phase-tracing variant")
    ap.add_argument("--debug", action="store_true",
                    help="build the variant whose kernels check metadata indices (FA_DEBUG)")
    a = ap.parse_args(argv)
    print(build(a.verbose, a.ptxas_info, a.force, a.trace, a.debug))
    return 0


if __name__ == "__main__":
    sys.exit(main())
