"""Builds libswb_moe.so in place: every .cu under csrc/ for sm_100a only."""
from __future__ import annotations

import glob
import os
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(_HERE, "libswb_moe.so")
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden"]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(_HERE, "csrc", "*.cu")))


def headers() -> list[str]:
    inc = os.path.join(os.path.dirname(_HERE), "include", "moe.h")
    return sorted(glob.glob(os.path.join(_HERE, "csrc", "*.h")) +
                  glob.glob(os.path.join(_HERE, "csrc", "*.cuh"))) + [inc]


def _stale() -> bool:
    if not os.path.exists(SO):
        return True
    t = os.path.getmtime(SO)
    return any(os.path.getmtime(f) > t for f in sources() + headers())


def build(force: bool = False, verbose_ptxas: bool = False, jobs: int = 8) -> str:
    if not (force or _stale()):
        return SO
    objdir = os.path.join(_HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    procs, objs = [], []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        objs.append(obj)
        procs.append(subprocess.Popen(["nvcc", *NVCC_FLAGS, *extra, "-c", src, "-o", obj]))
        while len([p for p in procs if p.poll() is None]) >= jobs:
            procs[0].wait()
    for p in procs:
        if p.wait() != 0:
            raise RuntimeError("nvcc failed")
    tmp = SO + ".tmp%d" % os.getpid()
    subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                           "-o", tmp, *objs, "-lcudart_static", "-ldl", "-lrt", "-lpthread"])
    os.replace(tmp, SO)
    return SO


if __name__ == "__main__":
    import sys
    build(force=True, verbose_ptxas="-v" in sys.argv)
    print(SO)
