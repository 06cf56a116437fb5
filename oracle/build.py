"""Build the C oracle (test infrastructure only; see oracle/__init__.py).

Compiles oracle/ppo.c with the host C compiler into oracle/libppo.so.
Building the checker is not using it: only tests, the smoke check and the
bench's CPU-baseline leg load the result.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ppo.c")
LIB = os.path.join(HERE, "libppo.so")


def build(force: bool = False) -> str:
    """Compile libppo.so if it is missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
           "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
