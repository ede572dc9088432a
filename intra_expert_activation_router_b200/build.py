"""Build the CUDA library libmoe_sparse.so in-tree, for sm_100a only.

    python -m intra_expert_activation_router_b200.build [-v]

Each .cu under csrc/ is compiled to an object in parallel (nvcc, -O3,
-gencode arch=compute_100a,code=sm_100a, -lineinfo, static CUDA runtime) and
the objects are linked into intra_expert_activation_router_b200/libmoe_sparse.so.
``-v`` adds ``-Xptxas -v`` (registers, spills, shared memory per kernel).
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT = os.path.join(PKG, "libmoe_sparse.so")
BUILD = os.path.join(ROOT, "_build")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmoe_sparse.so")


def flags(verbose: bool = False) -> list[str]:
    f = ["-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "-I", os.path.join(ROOT, "include"), "--expt-relaxed-constexpr"]
    if verbose:
        f += ["-Xptxas", "-v"]
    return f


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _up_to_date(srcs) -> bool:
    if not os.path.exists(OUT):
        return False
    deps = srcs + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(ROOT, "include", "moe_sparse.h"), __file__]
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(p) <= t for p in deps)


def build(verbose: bool = False, force: bool = False) -> str:
    srcs = sources()
    if not force and not verbose and _up_to_date(srcs):
        return OUT
    os.makedirs(BUILD, exist_ok=True)
    cc = nvcc()
    fl = flags(verbose)

    def compile_one(src):
        obj = os.path.join(BUILD, os.path.basename(src) + ".o")
        r = subprocess.run([cc, *fl, "-c", src, "-o", obj], capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stdout + r.stderr

    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(compile_one, srcs))
    if verbose:
        for _, log in results:
            sys.stdout.write(log)
    objs = [o for o, _ in results]
    tmp = OUT + ".tmp"
    r = subprocess.run([cc, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs],
                       capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force="-f" in sys.argv))
