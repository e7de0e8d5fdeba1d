"""Build step for the CPU oracle (test infrastructure only).

Compiles ``tlc_oracle.c`` into ``libtlc_oracle.so`` beside it with gcc:
single-threaded, -O2, IEEE fp32 on SSE, no FMA contraction, no fast-math.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-msse2", "-mfpmath=sse", "-Wall", "-Wextra"]


def oracle_library_path() -> str:
    return os.path.join(HERE, "libtlc_oracle.so")


def build_oracle(cc: str = "gcc") -> str:
    out = oracle_library_path()
    tmp = out + f".tmp{os.getpid()}"
    cmd = [cc, *CFLAGS, "-o", tmp, os.path.join(HERE, "tlc_oracle.c"), "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build_oracle())
