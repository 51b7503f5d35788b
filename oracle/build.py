"""Builds the fp64 oracle (``liboracle.so``) with gcc.  Test infrastructure."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "amk_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(out: str = LIB, defines=(), force: bool = False) -> str:
    """Compile ``amk_oracle.c`` into ``out`` (skipped when up to date)."""
    if (not force and not defines and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(SRC)):
        return out
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-Wall", "-Wextra", "-Wno-unused-parameter"]
    cmd += [f"-D{d}" for d in defines]
    tmp = out + f".tmp{os.getpid()}"
    cmd += ["-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
