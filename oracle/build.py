"""Compile the CPU oracle (test infrastructure) into oracle/liboracle.so.

The oracle is plain C: gcc, -O2, OpenMP over independent rows, and
-ffp-contract=off so that every fp32 multiply and add stays a separately
rounded operation.  No fast-math.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "w8a8_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def compile_lib(src: str, out: str) -> str:
    """Compile an oracle source file into a shared library (also used by the
    mutation test, which compiles deliberately altered copies)."""
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-std=gnu11", "-Wall", "-Wextra", "-shared", "-fPIC",
           "-o", out + ".tmp", src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    return compile_lib(SRC, LIB)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
