"""Compile the CPU oracle (``bitlinear_oracle.c``) into ``liboracle.so``.

Test infrastructure: the oracle is built so that the tests, the smoke check and
the benchmark's CPU-baseline leg can call it.  Plain gcc, no fast-math and no
floating-point contraction, so every operation is the IEEE operation written in
the source.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bitlinear_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
LIB_OMP = os.path.join(HERE, "liboracle_omp.so")  # the same source with OpenMP on

CFLAGS = ["-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-Wall", "-Wextra", "-Werror", "-Wno-unknown-pragmas"]


def _build_one(lib, extra, force):
    if (not force and os.path.exists(lib)
            and os.path.getmtime(lib) >= os.path.getmtime(SRC)):
        return lib
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, *extra, "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False) -> str:
    """Build liboracle.so (and its OpenMP twin liboracle_omp.so) if missing or
    older than the source; return the path of the plain one."""
    _build_one(LIB_OMP, ["-fopenmp"], force)
    return _build_one(LIB, [], force)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
