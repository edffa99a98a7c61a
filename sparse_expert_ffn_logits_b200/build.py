"""Builds libsparse_moe.so, the C-ABI library of hand-written sm_100a kernels, in-tree."""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
INCLUDE = os.path.join(ROOT, "include")
SO = os.path.join(HERE, "libsparse_moe.so")
OBJ = os.path.join(ROOT, "_build", "sparse_moe")
SOURCES = ["moe_api.cu", "router.cu", "gate.cu", "select.cu", "updown.cu", "layer.cu", "misc.cu",
           "route_noalloc.cu", "dense.cu"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
              "-Xcompiler", "-fPIC", "-I", INCLUDE, "-Xptxas", "-warn-spills"]


def _deps():
    return ([os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "moe.h")])


def _stale():
    if not os.path.exists(SO):
        return True
    t = os.path.getmtime(SO)
    return any(os.path.getmtime(d) > t for d in _deps())


def build(force=False, verbose=False, extra_flags=()):
    if not force and not _stale():
        return SO
    os.makedirs(OBJ, exist_ok=True)
    flags = NVCC_FLAGS + list(extra_flags) + (["-Xptxas", "-v"] if verbose else [])

    def compile_one(src):
        obj = os.path.join(OBJ, src.replace(".cu", ".o"))
        r = subprocess.run(["nvcc", *flags, "-c", os.path.join(CSRC, src), "-o", obj],
                           capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stderr

    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(compile_one, SOURCES))
    if verbose:
        for _, log in results:
            sys.stderr.write(log)
    objs = [o for o, _ in results]
    subprocess.check_call(["nvcc", "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-o", SO, *objs])
    return SO


if __name__ == "__main__":
    build(force=True, verbose="-v" in sys.argv)
