"""Build ``libw4.so`` (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

    python -m bit_gemm_wise_b200.build [--force]

Every translation unit is compiled with ``-gencode arch=compute_100a,code=sm_100a
-lineinfo -O3``; the quantizer and the activation quantizer additionally with
``-fmad=false`` (their codes must be bit-identical to a plain IEEE evaluation). No
fast-math anywhere. Objects go to ``_build/`` and the library next to this file.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libw4.so")

SOURCES = {
    "w4_abi.cu": [],
    "w4_quantize.cu": ["-fmad=false"],
    "fp8_row_quant.cu": ["-fmad=false"],
    "w4_prepack.cu": [],
    "w4a16_gemv.cu": [],
    "w4a16_tc.cu": [],
    "w4a8_gemm.cu": [],
    "w4_moe.cu": [],
    "w4_nf4.cu": [],
}

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
          "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _stale(obj: str, deps: list[str]) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    headers.append(os.path.join(INCLUDE, "w4.h"))
    objs = []
    for src, extra in SOURCES.items():
        path = os.path.join(CSRC, src)
        if not os.path.exists(path):
            continue
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(obj)
        if force or _stale(obj, [path] + headers + [__file__]):
            cmd = [nvcc(), *ARCH, *COMMON, *extra, "-c", path, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
                print(" ".join(cmd), flush=True)
            subprocess.check_call(cmd)
    if force or _stale(LIB, objs):
        tmp = LIB + ".tmp"
        subprocess.check_call([nvcc(), *ARCH, "-shared", "-o", tmp, *objs])
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
