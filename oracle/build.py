"""Compile the plain-C oracle into oracle/libdq_oracle.so.

TEST INFRASTRUCTURE: the oracle is built by ``__graft_entry__.build()`` and
loaded only by tests/, ``__graft_entry__.smoke()`` and bench.py's
cpu_baseline/reference legs. Building it is not using it.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "dq_oracle.c")
HDR = os.path.join(HERE, "dq_oracle.h")
LIB = os.path.join(HERE, "libdq_oracle.so")

# -ffp-contract=off: no fused multiply-add, so every fp32 product and sum in
# the encoder is rounded on its own, as the format defines.
CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
          "-shared", "-Wall", "-Wextra", "-D_DEFAULT_SOURCE"]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in (SRC, HDR, __file__))


def build(force: bool = False) -> str:
    if force or needs_build():
        tmp = LIB + ".tmp.%d" % os.getpid()
        cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
