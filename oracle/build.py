"""Compile the oracle's C arithmetic into ``oracle/libzero_oracle.so``.

Flags keep every operation a single IEEE-754 operation: no contraction of
multiply-add, no fast-math, no flush of subnormals.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def build(verbose: bool = False, src: str = None, out: str = None) -> str:
    src = src or os.path.join(HERE, "zero_oracle.c")
    out = out or os.path.join(HERE, "libzero_oracle.so")
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-fno-finite-math-only", "-frounding-math", "-Wall", "-Wextra", "-o", out, src, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(verbose=True))
