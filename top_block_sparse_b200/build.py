"""Builds libsa.so (the sm_100a kernels and the C ABI) in-tree with nvcc.

    python -m top_block_sparse_b200.build [--verbose] [--force]

Objects go to top_block_sparse_b200/_build/, the library to
top_block_sparse_b200/libsa.so.  The CUDA runtime is linked statically so the
library loads on machines without a GPU (symbol checks) and needs nothing
besides the driver on a GPU machine.
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
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libsa.so")
INCLUDE = os.path.join(ROOT, "include")

SOURCES = ["sa_api.cu", "pool.cu", "score_topk.cu", "decode_attn.cu", "decode_tc.cu", "prefill_score.cu", "prefill_attn.cu", "verify.cu", "bucket.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps_mtime() -> float:
    names = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    names.append(os.path.join(INCLUDE, "sa.h"))
    names.append(os.path.abspath(__file__))
    return max(os.path.getmtime(n) for n in names)


def _compile(src: str, force: bool, verbose: bool, ptxas_v: bool) -> tuple[str, str]:
    obj = os.path.join(BUILD, src.replace(".cu", ".o"))
    path = os.path.join(CSRC, src)
    if (not force and os.path.exists(obj)
            and os.path.getmtime(obj) >= max(os.path.getmtime(path), _deps_mtime())):
        return obj, ""
    cmd = [nvcc(), *ARCH, *FLAGS, "-c", path, "-o", obj]
    if ptxas_v:
        cmd[1:1] = ["-Xptxas", "-v"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def build(force: bool = False, verbose: bool = False, ptxas_v: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(lambda s: _compile(s, force, verbose, ptxas_v), SOURCES))
    objs = [o for o, _ in results]
    if ptxas_v:
        for (_, log), src in zip(results, SOURCES):
            if log:
                print(f"== {src}\n{log}")
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs):
        tmp = LIB + ".tmp"
        cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print registers / spills / shared memory")
    a = ap.parse_args(argv)
    print(build(a.force, a.verbose, a.ptxas_v))
    return 0


if __name__ == "__main__":
    sys.exit(main())
