"""Compiles the CPU oracle (test infrastructure) into oracle/_ep_oracle.so.

gcc, -O2, -ffp-contract=off and no fast-math: every float operation of the
oracle is one IEEE binary32 operation in the written order."""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ep_oracle.c")
LIB = os.path.join(HERE, "_ep_oracle.so")
SELFTEST = os.path.join(HERE, "selftest.c")
FLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wextra"]


def compile_to(src: str, out: str) -> str:
    """Compiles an oracle source file with the oracle's flags."""
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", *FLAGS, "-fPIC", "-shared", "-fvisibility=hidden", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def compile_selftest(out: str) -> str:
    """The oracle's C self-test (hand-derived values) as an executable."""
    subprocess.run(["gcc", *FLAGS, "-Werror", "-o", out, SELFTEST, "-lm"], check=True)
    return out


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    return compile_to(SRC, LIB)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
