"""Build the in-tree CUDA library ``libsherry.so`` for sm_100a (B200).

Run ``python -m sparse_ternary_weight_b200.build`` (or ``build()``).  Each .cu
file is compiled separately with nvcc (no fast-math: the scale path relies on
IEEE division and no flush-to-zero) and linked into one shared library with a
plain C ABI (include/sherry.h).
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libsherry.so")
OBJ = os.path.join(ROOT, "_build")

SOURCES = ["api.cu", "quantize.cu", "unpack.cu", "gemv.cu", "gemv_stream.cu", "gemv_mma.cu", "gemv_tc.cu", "prefill.cu", "noalloc.cu", "tequila.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--ftz=false", "--prec-div=true",
          "--prec-sqrt=true", "-I", os.path.join(ROOT, "include")]
PER_FILE = {"quantize.cu": ["--fmad=false"], "tequila.cu": ["--fmad=false"]}


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(OBJ, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    headers.append(os.path.join(ROOT, "include", "sherry.h"))
    objs = []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(OBJ, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _stale(o, [s, *headers, __file__]):
            cmd = [nvcc(), *ARCH, *COMMON, *PER_FILE.get(src, []), "-c", s, "-o", o]
            if verbose:
                cmd.append("-Xptxas=-v")
                print(" ".join(cmd), flush=True)
            subprocess.run(cmd, check=True)
    if force or _stale(OUT, objs):
        cmd = [nvcc(), *ARCH, "-shared", "-o", OUT + ".tmp", *objs, "-lcudart"]
        subprocess.run(cmd, check=True)
        os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(OUT)
