"""Compile the C oracle into oracle/_build/libnvfp4_oracle.so.

Test infrastructure: the oracle is built (never imported) by the package build step and
loaded only by the tests, the smoke check and the bench's CPU-baseline leg.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "libnvfp4_oracle.so")
SOURCES = [os.path.join(HERE, "nvfp4_oracle.c")]
HEADERS = [os.path.join(HERE, "nvfp4_oracle.h")]

# IEEE binary32 semantics: no fast-math, no contraction of a*b+c into fma, SSE math (x86-64).
CFLAGS = ["-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
          "-Wall", "-Wextra"]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in SOURCES + HEADERS + [__file__])


def build(force: bool = False) -> str:
    if force or not up_to_date():
        os.makedirs(OUT_DIR, exist_ok=True)
        tmp = LIB + ".tmp"
        cmd = ["gcc", *CFLAGS, *SOURCES, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
