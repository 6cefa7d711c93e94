"""Builds the CPU oracle (test infrastructure) into oracle/liboracle.so.

The oracle is plain C99 compiled with gcc; it shares nothing with the CUDA
library.  Run as a script or call build().
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ssmq_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile ssmq_oracle.c if the shared library is missing or stale."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(SRC),
                                             os.path.getmtime(os.path.join(HERE, "ssmq_oracle.h")))):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    # -O2 without -ffast-math: IEEE semantics (division, rounding, NaN tests)
    # are part of the oracle's definition.  -ffp-contract=off keeps every
    # multiply-add a separately rounded pair, as written.
    cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-o", tmp, SRC, "-lm", "-lpthread"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
