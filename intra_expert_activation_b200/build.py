"""Build libmoe_sparse.so (the C-ABI library) in-tree for sm_100a with nvcc.

    python -m intra_expert_activation_b200.build [--force] [-v] [--check]

--check builds libmoe_sparse_check.so instead: the same library with the
kernels' bounds checks on the data-derived indices compiled in
(-DMOE_CHECK=1; a failed check sets MOE_ERR_INVALID in the status word). The
binding loads it when MOE_SPARSE_LIB=check is set in the environment.

Objects go to _build/ at the repository root; the shared library is written
next to this file so that the Python binding loads it from the package.
"""

from __future__ import annotations

import argparse
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmoe_sparse.so")
LIB_CHECK = os.path.join(PKG, "libmoe_sparse_check.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
         "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    hs += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return hs


def _mtime(p):
    return os.path.getmtime(p) if os.path.exists(p) else -1.0


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          check: bool = False) -> str:
    out_dir = os.path.join(BUILD, "check") if check else BUILD
    lib = LIB_CHECK if check else LIB
    flags = FLAGS + (["-DMOE_CHECK=1"] if check else [])
    os.makedirs(out_dir, exist_ok=True)
    hdr_t = max(_mtime(h) for h in headers())
    objs, jobs = [], []
    for src in sources():
        obj = os.path.join(out_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or _mtime(obj) < max(_mtime(src), hdr_t):
            cmd = [nvcc(), *ARCH, *flags, "-c", src, "-o", obj]
            if ptxas_info:
                cmd += ["-Xptxas", "-v"]
            jobs.append(cmd)

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0 or verbose or ptxas_info:
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed: {' '.join(cmd)}")

    with ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as pool:
        list(pool.map(run, jobs))
    if jobs or not os.path.exists(lib) or _mtime(lib) < max(_mtime(o) for o in objs):
        cmd = [nvcc(), *ARCH, "-shared", "-o", lib, *objs, "-lcudart_static", "-lrt", "-ldl",
               "-lpthread"]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("link failed")
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    ap.add_argument("--check", action="store_true", help="bounds-checked build (MOE_CHECK=1)")
    a = ap.parse_args()
    print(build(a.force, a.verbose, a.ptxas_info, a.check))
