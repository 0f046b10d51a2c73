"""Builds libep.so (the C-ABI library of csrc/) in-tree with nvcc for sm_100a.

    python -m combine_topk_idx_rank_b200.build [--force] [--verbose]

``--verbose`` passes -Xptxas -v (registers, spills, shared memory per kernel).
The CUDA runtime is linked statically, so the library needs only the driver.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libep.so")
OBJDIR = os.path.join(HERE, "_build")
SOURCES = ["routing.cu", "pack.cu", "combine.cu", "gating.cu", "padding.cu", "peer.cu", "ep_api.cu", "ep_noalloc.cu"]
HEADERS = ["ep_internal.cuh", "quant.cuh", "tma.cuh", os.path.join("..", "..", "include", "ep.h"),
           os.path.join("..", "..", "include", "ep_testing.h")]

NVCC = os.environ.get("NVCC", "nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include")]


def _mtime(p):
    return os.path.getmtime(p) if os.path.exists(p) else 0.0


def build(force: bool = False, verbose: bool = False) -> str:
    deps = [os.path.join(CSRC, s) for s in SOURCES] + [os.path.join(CSRC, h) for h in HEADERS]
    if not force and _mtime(LIB) >= max(_mtime(d) for d in deps):
        return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    objs = []
    for s in SOURCES:
        obj = os.path.join(OBJDIR, s.replace(".cu", ".o"))
        cmd = [NVCC, *FLAGS, "-c", os.path.join(CSRC, s), "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = LIB + ".tmp"
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs,
                    "-cudart", "static"], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
