"""Build libmxattn.so in place with nvcc for sm_100a.

    python -m mxfp4_bit_attention_b200.build [--force] [--verbose]

Each .cu file is compiled to an object (cached by modification time) and the
objects are linked into ``mxfp4_bit_attention_b200/libmxattn.so`` against the
CUDA runtime.  ``--verbose`` adds ``-Xptxas -v`` (registers, spills, shared
memory per kernel).
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
OUT = os.path.join(HERE, "libmxattn.so")
SOURCES = ["api.cu", "quant.cu", "attn.cu", "attn_wide.cu", "probe.cu", "noalloc.cu", "sweep.cu", "varlen.cu"]
HEADERS = ["ptx.cuh", "kernels.cuh"]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else (shutil.which("nvcc") or "nvcc")


FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr"]


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    deps = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "mxattn.h")]
    dep_time = max(os.path.getmtime(p) for p in deps)
    objs = []
    for src in SOURCES:
        sp = os.path.join(CSRC, src)
        op = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(op)
        if force or verbose or not os.path.exists(op) or os.path.getmtime(op) < max(os.path.getmtime(sp), dep_time):
            cmd = [nvcc(), *FLAGS, "-I", os.path.join(ROOT, "include"), "-c", sp, "-o", op]
            if verbose:
                cmd += ["-Xptxas", "-v"]
            subprocess.run(cmd, check=True)
    if force or not os.path.exists(OUT) or os.path.getmtime(OUT) < max(os.path.getmtime(o) for o in objs):
        subprocess.run([nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-cudart", "static",
                        "-o", OUT, *objs], check=True)
    return OUT


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    args = ap.parse_args()
    print(build(args.force, args.verbose), file=sys.stderr)
