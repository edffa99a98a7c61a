"""Builds the seeded input generator: libsynth_host.so (g++) and libsynth_cuda.so (nvcc, sm_100a)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SO = os.path.join(HERE, "libsynth_host.so")
CUDA_SO = os.path.join(HERE, "libsynth_cuda.so")


def _stale(target, sources):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build_host(force=False):
    srcs = [os.path.join(HERE, "synth_host.cpp"), os.path.join(HERE, "synth.h")]
    if force or _stale(HOST_SO, srcs):
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-pthread", "-o", HOST_SO, srcs[0]])
    return HOST_SO


def build_cuda(force=False):
    srcs = [os.path.join(HERE, "synth_cuda.cu"), os.path.join(HERE, "synth.h")]
    if force or _stale(CUDA_SO, srcs):
        subprocess.check_call(["nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
                               "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
                               "-o", CUDA_SO, srcs[0]])
    return CUDA_SO


def build(force=False):
    build_host(force)
    build_cuda(force)


if __name__ == "__main__":
    build(force=True)
