"""Compile the C oracle into ``oracle/libgauss_oracle.so``.

Test infrastructure only (see ``gauss_oracle.c``).  Plain ``gcc -O2 -fopenmp``:
no fast-math, so every double operation keeps IEEE semantics and the result of
one row does not depend on the thread count.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gauss_oracle.c")
LIB = os.path.join(HERE, "libgauss_oracle.so")


def build_oracle(out=LIB, extra_flags=(), force=False):
    """Build the oracle shared library; return its path."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(SRC)
            and not extra_flags):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
           "-ffp-contract=off", "-fexcess-precision=standard", *extra_flags, SRC, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build_oracle(force="--force" in sys.argv))
