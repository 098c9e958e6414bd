"""Builds the two generator libraries in place (host: gcc, GPU: nvcc sm_100a)."""
from __future__ import annotations

import os
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))
CPU_SO = os.path.join(_HERE, "libmoegen_cpu.so")
GPU_SO = os.path.join(_HERE, "libmoegen_gpu.so")


def _stale(out: str, srcs: list[str]) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(s) > t for s in srcs)


def build_cpu(force: bool = False) -> str:
    src = os.path.join(_HERE, "csrc", "philox_cpu.c")
    if force or _stale(CPU_SO, [src]):
        tmp = CPU_SO + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, src, "-lm"])
        os.replace(tmp, CPU_SO)
    return CPU_SO


def build_gpu(force: bool = False) -> str:
    src = os.path.join(_HERE, "csrc", "philox_gpu.cu")
    if force or _stale(GPU_SO, [src]):
        tmp = GPU_SO + ".tmp%d" % os.getpid()
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                               "-lineinfo", "-fmad=false", "-Xcompiler", "-fPIC", "-shared",
                               "-o", tmp, src])
        os.replace(tmp, GPU_SO)
    return GPU_SO


def build_all(force: bool = False) -> None:
    build_cpu(force)
    build_gpu(force)
