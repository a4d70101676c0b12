"""Build the test-only probes: tests/probe/_build/libcvtprobe.so (hardware conversions) and
tests/probe/_build/libbarrierprobe.so (the one-launch quantizer with a chosen barrier count)."""
import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
SRC = os.path.join(HERE, "cvt_probe.cu")
LIB = os.path.join(HERE, "_build", "libcvtprobe.so")
BARRIER_SRC = os.path.join(HERE, "barrier_probe.cu")
BARRIER_LIB = os.path.join(HERE, "_build", "libbarrierprobe.so")


def _nvcc(src: str, lib: str, deps=(), force: bool = False) -> str:
    newest = max([os.path.getmtime(p) for p in (src, *deps)])
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < newest:
        os.makedirs(os.path.dirname(lib), exist_ok=True)
        subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                        "-std=c++17", "-fmad=false", "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
                        "-shared", "-Xcompiler", "-fPIC", "-cudart", "static", src, "-o", lib + ".tmp"], check=True)
        os.replace(lib + ".tmp", lib)
    return lib


def build(force: bool = False) -> str:
    return _nvcc(SRC, LIB, force=force)


def build_barrier(force: bool = False) -> str:
    deps = glob.glob(os.path.join(ROOT, "nvfp4_block_scaled_13_b200", "csrc", "*.cuh"))
    deps.append(os.path.join(ROOT, "include", "nvfp4.h"))
    return _nvcc(BARRIER_SRC, BARRIER_LIB, deps, force=force)


if __name__ == "__main__":
    print(build(force=True))
    print(build_barrier(force=True))
