"""Builds the CPU oracle (plain C) with gcc: oracle/liboracle.so
(single-threaded) and, from the same source with -fopenmp,
oracle/liboracle_omp.so (token loops split across threads).

Test infrastructure: the oracle is only used by the tests, the smoke check and
the benchmark's CPU-baseline leg.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ep_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
LIB_OMP = os.path.join(HERE, "liboracle_omp.so")

# -ffp-contract=off: no compiler-fused multiply-adds beyond the explicit fmaf
# calls, so every float operation rounds exactly as written.
CFLAGS = ["-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-Wall", "-Wextra", "-Wno-unused-parameter", "-Wno-unknown-pragmas"]


def _build_one(lib: str, extra, force: bool) -> str:
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= os.path.getmtime(SRC):
        return lib
    # -Bsymbolic: calls between the oracle's own functions stay inside this
    # library when both builds are loaded in one process
    cmd = ["gcc", *CFLAGS, *extra, "-Wl,-Bsymbolic", "-o", lib + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


def build(force: bool = False) -> str:
    """Builds both libraries; returns the single-threaded one."""
    _build_one(LIB_OMP, ["-fopenmp"], force)
    return _build_one(LIB, [], force)


def build_omp(force: bool = False) -> str:
    return _build_one(LIB_OMP, ["-fopenmp"], force)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
