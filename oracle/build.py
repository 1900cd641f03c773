"""Build the CPU oracle shared library (test infrastructure only).

    python -m oracle.build          # or oracle.build.build()

Compiles ``lynx_oracle.c`` with gcc into ``oracle/_build/liblynx_oracle.so``.
Floating point is neither contracted (no FMA) nor reassociated, so every fp32
operation in the oracle is one IEEE-rounded operation.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lynx_oracle.c")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "liblynx_oracle.so")

FLAGS = ["-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
         "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile the oracle if the source is newer than the library; return its path."""
    os.makedirs(OUT_DIR, exist_ok=True)
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", *FLAGS, "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
