"""Builds the CPU oracle's shared library (test infrastructure only).

The oracle is plain C compiled with gcc at -O2 without -ffast-math, so the
compiler keeps the order of every floating-point operation as written.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "gdn_oracle.c")
LIBRARY = os.path.join(HERE, "libgdn_oracle.so")


def build(force: bool = False) -> str:
    """Compiles gdn_oracle.c into libgdn_oracle.so next to it; returns its path."""
    if (not force and os.path.exists(LIBRARY)
            and os.path.getmtime(LIBRARY) >= os.path.getmtime(SOURCE)):
        return LIBRARY
    tmp = LIBRARY + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-std=c11",
           "-Wall", "-Wextra", "-o", tmp, SOURCE]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIBRARY)
    return LIBRARY


if __name__ == "__main__":
    print(build(force=True))
