"""Build libqlora.so (sm_100a) in-tree with nvcc.

    python -m bit_quantized_lora_blockwise_b200.build

One translation unit (csrc/qlora.cu); the CUDA runtime is linked
statically, the driver's cuTensorMapEncodeTiled is looked up at run time, so
the library needs nothing beyond the NVIDIA driver. No fast-math: the codec
is bit-exact only under IEEE fp32 division and round-to-nearest conversions.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libqlora.so")
SOURCES = ["qlora.cu", "codec.cuh", "gemm.cuh", "skinny.cuh", "smallm.cuh", "adamw.cuh", "ptx.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str = LIB, verbose_ptxas: bool = False) -> list[str]:
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-prec-div=true", "-prec-sqrt=true", "-ftz=false",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           "-o", out, os.path.join(CSRC, "qlora.cu")]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + [os.path.join(ROOT, "include", "qlora.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if force or needs_build():
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(command(tmp, verbose_ptxas))
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose_ptxas="-v" in sys.argv)
    print(LIB)
