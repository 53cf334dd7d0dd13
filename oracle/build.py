"""Compile the fp64 CPU oracle (``kda_oracle.c``) into ``libkda_oracle.so``.

Test infrastructure: the oracle checks the CUDA library; it is never part of
the product path. ``python oracle/build.py`` or ``oracle.build.build()``.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kda_oracle.c")
LIB = os.path.join(HERE, "libkda_oracle.so")


def build(force: bool = False) -> str:
    """Build the oracle library if it is missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    # -O2 without -ffast-math: IEEE fp64, sums in index order, no contraction
    # into fused multiply-adds, so the result is the plain definition.
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
           "-o", tmp, SRC, "-lm", "-lpthread"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
