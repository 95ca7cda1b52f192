"""Build the float64 oracle (oracle.c, moshi_streams.c) into oracle/liboracle.so with gcc + OpenMP.

Test infrastructure: building the checker is not using it. -ffp-contract=off keeps
every multiply and add a separate IEEE operation, as the source reads.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(HERE, "liboracle.so")


def sources() -> list:
    return [os.path.join(HERE, "oracle.c"), os.path.join(HERE, "moshi_streams.c")]


def build_oracle(verbose: bool = False) -> str:
    out = library_path()
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fopenmp", "-ffp-contract=off",
           "-fPIC", "-shared", "-o", tmp, *sources(), "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build_oracle(verbose=True))
