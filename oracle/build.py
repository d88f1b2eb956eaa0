"""Compile the oracle (plain C) into ``oracle/libecho_oracle.so``.

Test infrastructure: the library this builds is loaded only by the tests, the
package smoke check and the benchmark's CPU-baseline leg.

The flags keep every binary32 operation a separate IEEE operation:
``-ffp-contract=off`` (no fused multiply-add), no ``-ffast-math``, and x86-64
SSE arithmetic (the default on that target). ``-fopenmp`` is not used: the
oracle is single-threaded; callers that want parallel timing split the group
columns across processes.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "echo_oracle.c")
LIB = os.path.join(HERE, "libecho_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = [
        os.environ.get("CC", "gcc"),
        "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
        "-fno-unsafe-math-optimizations", "-frounding-math",
        "-Wall", "-Wextra", "-fPIC", "-shared",
        SRC, "-o", LIB + ".tmp", "-lm",
    ]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
