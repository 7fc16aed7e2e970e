"""Compile the CPU oracle (qmv_oracle.c) into oracle/liboracle.so.

Test infrastructure: the product library never links this.  Flags keep every
floating-point operation IEEE-exact in source order (no contraction, no fast
math), so the oracle's results do not depend on the compiler's scheduling.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "qmv_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    flags = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
             "-fno-unsafe-math-optimizations", "-fPIC", "-shared", "-Wall",
             "-Wextra", "-Wno-unused-parameter"]
    # Row-parallel OpenMP (bit-identical results: rows are independent) when
    # the compiler has it, else a serial build.
    compilers = [c for c in ("/usr/bin/gcc", os.environ.get("CC"), "gcc") if c]
    last = None
    for cc in compilers:
        for omp in (["-fopenmp"], []):
            cmd = [cc] + flags + omp + [SRC, "-o", LIB + ".tmp", "-lm"]
            if verbose:
                print(" ".join(cmd), file=sys.stderr)
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode == 0:
                os.replace(LIB + ".tmp", LIB)
                return LIB
            last = r.stderr
    raise RuntimeError("cannot build the oracle:\n" + (last or ""))


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
