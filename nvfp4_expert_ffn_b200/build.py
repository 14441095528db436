"""Build libmoe_nvfp4.so (all CUDA sources, sm_100a) in-tree.

    python -m nvfp4_expert_ffn_b200.build [--jobs N]

Objects go to <repo>/_build/, the library to nvfp4_expert_ffn_b200/lib/.

    python -m nvfp4_expert_ffn_b200.build --trace

builds a separate library with the FFN kernel's timeline trace compiled in
(<repo>/_build/trace/libmoe_nvfp4_trace.so); load it by setting MOE_NVFP4_LIB to its path.
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
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libmoe_nvfp4.so")
BUILD = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-std=c++17", "-Xcompiler", "-fPIC",
                     "-Xptxas", "-v", "-I", os.path.join(ROOT, "include"), "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _compile(src: str, outdir: str = BUILD, extra: tuple = ()) -> tuple[str, str]:
    obj = os.path.join(outdir, os.path.basename(src) + ".o")
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
    with open(obj + ".ptxas.txt", "w") as f:
        f.write(r.stderr)
    return obj, r.stderr


def build(jobs: int = 8, verbose: bool = False, trace: bool = False) -> str:
    outdir = os.path.join(BUILD, "trace") if trace else BUILD
    lib = os.path.join(outdir, "libmoe_nvfp4_trace.so") if trace else LIB
    extra = ("-DMOE_TRACE", "-lineinfo") if trace else ()
    os.makedirs(outdir, exist_ok=True)
    os.makedirs(LIBDIR, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        results = list(ex.map(lambda s: _compile(s, outdir, extra), srcs))
    objs = [o for o, _ in results]
    if verbose:
        for _, log in results:
            sys.stdout.write(log)
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--jobs", type=int, default=8)
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--trace", action="store_true", help="separate library with the FFN timeline trace")
    a = ap.parse_args()
    print(build(a.jobs, a.verbose, a.trace))
