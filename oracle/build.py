"""Build the fp64 CPU oracle (``liboracle.so``) with the host C compiler.

Test infrastructure only: the product library never links or loads it.
Run ``python oracle/build.py`` or call :func:`build`.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "swa_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def compile_lib(src: str, out: str) -> str:
    """Compile the C oracle source `src` into the shared library `out`."""
    # -O2 without -ffast-math keeps IEEE fp64 semantics and the written order.
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-o", out + ".tmp", src, "-lm"]
    subprocess.check_call(cmd)
    os.replace(out + ".tmp", out)
    return out


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    return compile_lib(SRC, LIB)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
