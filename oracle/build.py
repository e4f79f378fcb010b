"""Build the fp64 CPU oracle shared library (test infrastructure only).

    python oracle/build.py            # writes oracle/libmh3a_oracle.so

Plain gcc, -O3, OpenMP.  The oracle is the checker: it is compiled here but never linked
into, imported by or called from the CUDA library.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mh3a_oracle.c")
LIB = os.path.join(HERE, "libmh3a_oracle.so")


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the oracle if the library is missing or older than its sources."""
    deps = [SRC, os.path.join(HERE, "mh3a_oracle.h")]
    if not force and os.path.exists(LIB) and all(
        os.path.getmtime(LIB) >= os.path.getmtime(d) for d in deps
    ):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    # x86-64-v3 (AVX2/FMA) keeps the library portable across the hosts it is copied to;
    # -ffp-contract=off keeps each multiply and add a separately rounded fp64 operation.
    cmd = [
        "gcc", "-O3", "-march=x86-64-v3", "-ffp-contract=off", "-fopenmp", "-fPIC",
        "-shared", "-std=c11", "-Wall", "-o", tmp, SRC, "-lm",
    ]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
