"""Compile the CPU oracle into oracle/liboracle.so (gcc, OpenMP).

Test infrastructure: the tests, the smoke check and the benchmark's CPU
baseline load the result; the CUDA library never does.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
OUT = os.path.join(HERE, "liboracle.so")


def build(src: str = SRC, out: str = OUT, extra=()) -> str:
    if (src == SRC and out == OUT and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-Wall", "-Werror",
           *extra, src, "-o", out]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build())
    sys.exit(0)
