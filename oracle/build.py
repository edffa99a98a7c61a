"""Builds the fp64 CPU oracle, liboracle.so, with g++ (test infrastructure only)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "liboracle.so")
SRC = os.path.join(HERE, "oracle.cpp")


def compile_oracle(src, out, extra=()):
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
                           "-ffp-contract=off", "-fno-fast-math", *extra, "-o", out, src])
    return out


def build(force=False):
    if force or not os.path.exists(SO) or os.path.getmtime(SRC) > os.path.getmtime(SO):
        compile_oracle(SRC, SO)
    return SO


if __name__ == "__main__":
    build(force=True)
