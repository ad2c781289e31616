"""Build the CPU oracle (plain C, gcc) into ``oracle/liboracle.so``.

TEST INFRASTRUCTURE: the oracle is the checker, built beside the library but
never linked into it.  ``-ffp-contract=off`` keeps every fp32 product and sum
separately rounded, as the oracle's combine definition requires.
"""

import os
import subprocess
import sys

_HERE = os.path.dirname(os.path.abspath(__file__))


def oracle_lib_path(openmp: bool = False) -> str:
    return os.path.join(_HERE, "liboracle_omp.so" if openmp else "liboracle.so")


def build_oracle(verbose: bool = False, openmp: bool = False) -> str:
    """The plain single-threaded build (``liboracle.so``, what the tests
    check against) or, with ``openmp``, the same source with its row loops
    shared among the host cores (``liboracle_omp.so``, for the benchmark's
    CPU baseline only)."""
    src = os.path.join(_HERE, "moe_oracle.c")
    out = oracle_lib_path(openmp)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
           "-fexcess-precision=standard", "-fPIC", "-shared", "-Wall", "-Wextra"]
    cmd += ["-fopenmp"] if openmp else []
    cmd += ["-o", tmp, src, "-lm"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build_oracle(verbose=True))
    print(build_oracle(verbose=True, openmp=True))
