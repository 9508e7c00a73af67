"""Compile the C oracle (test infrastructure) into oracle/_build/liboracle.so.

Plain gcc, -O2, no intrinsics.  Building the checker is not using it; the
package build step calls this so that the oracle is ready on a fresh machine.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "dcn_oracle.c")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "liboracle.so")


def compile_oracle(src=SRC, lib=LIB, extra_flags=()):
    """Compile `src` into the shared object `lib`; returns the path."""
    os.makedirs(os.path.dirname(lib), exist_ok=True)
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-Wall", "-Werror",
           *extra_flags, src, "-o", lib, "-lm"]
    subprocess.run(cmd, check=True)
    return lib


def build(force=False):
    """Build the oracle library if it is missing or older than its source."""
    if (force or not os.path.exists(LIB)
            or os.path.getmtime(LIB) < os.path.getmtime(SRC)):
        compile_oracle()
    return LIB


if __name__ == "__main__":
    print(build(force=True))
