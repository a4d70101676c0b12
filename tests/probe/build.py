"""Build the test-only conversion probe (tests/probe/_build/libcvtprobe.so)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cvt_probe.cu")
LIB = os.path.join(HERE, "_build", "libcvtprobe.so")


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        os.makedirs(os.path.dirname(LIB), exist_ok=True)
        subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                        "-fmad=false", "-shared", "-Xcompiler", "-fPIC", "-cudart", "static", SRC,
                        "-o", LIB + ".tmp"], check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
