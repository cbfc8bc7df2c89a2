"""Build the in-tree CUDA library liblora_b200.so for sm_100a.

    python -m lora_adapter_execution_b200.build [--verbose]

Sources: csrc/lora_b200.cu (kernels + C ABI, one translation unit so the
device status word is a single symbol) and csrc/plan.cpp (host planner).
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "liblora_b200.so")
BUILD_DIR = os.path.join(ROOT, "_build")
SOURCES = [os.path.join(CSRC, "lora_b200.cu"), os.path.join(CSRC, "plan.cpp")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("common.cuh", "gemm.cuh", "skinny.cuh", "switch.cuh", "tsqr.cuh", "compress.cuh", "qr_api.inc", "internal.h")] + [
    os.path.join(ROOT, "include", "lora.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(d) > t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    objs = []
    common = ["-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include")]
    for src in SOURCES:
        obj = os.path.join(BUILD_DIR, os.path.basename(src) + ".o")
        if src.endswith(".cu"):
            cmd = [NVCC, *ARCH, "-lineinfo", *common, "-c", src, "-o", obj]
            if verbose:
                cmd += ["-Xptxas", "-v"]
        else:
            cmd = ["g++", "-O3", "-std=c++17", "-fPIC", "-I", os.path.join(ROOT, "include"), "-c", src, "-o", obj]
        subprocess.check_call(cmd)
        objs.append(obj)
    tmp = LIB + ".tmp"
    subprocess.check_call([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
