"""Compile the CPU oracle (plain C, gcc, OpenMP) into oracle/_build/liboracle.so.

Test infrastructure: building the checker is not using it.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pi_oracle.c")
BUILD_DIR = os.path.join(HERE, "_build")
LIB_PATH = os.path.join(BUILD_DIR, "liboracle.so")
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-Wall", "-Wextra", "-Wno-unused-parameter"]


def compile_to(src: str, out: str) -> None:
    os.makedirs(os.path.dirname(out), exist_ok=True)
    subprocess.run(["gcc", *CFLAGS, "-o", out, src, "-lm"], check=True)


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < os.path.getmtime(SRC):
        compile_to(SRC, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force=True))
