"""Build ``libmoe.so`` in-tree with nvcc for sm_100a (no GPU needed to build).

    python -m combine_moe_topk_gate_b200.build [--force] [--ptxas-verbose] [--bounds-check]

Each ``csrc/*.cu`` is compiled to an object file in ``_build/`` (in parallel),
then the objects are linked into the shared library with the CUDA runtime
linked statically.  ``--bounds-check`` builds ``libmoe_bounds_check.so``
instead: the same sources with ``-DMOE_BOUNDS_CHECK``, whose kernels also test
every receive-row index they compute themselves against the buffer's rows and
report one outside it through the status word (load it with
``MOE_LIBRARY=<path>``).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmoe.so")
LIB_BOUNDS_CHECK = os.path.join(PKG, "libmoe_bounds_check.so")
OBJ_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-fmad=false", "-Xcompiler", "-fPIC",
                 "-I", INCLUDE, "-I", CSRC]
LINK_FLAGS = [*ARCH, "-shared", "-cudart", "static"]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps() -> list[str]:
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + [os.path.join(INCLUDE, "moe.h"), __file__]


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


def build(force: bool = False, ptxas_verbose: bool = False, bounds_check: bool = False) -> str:
    lib = LIB_BOUNDS_CHECK if bounds_check else LIB
    if not (force or ptxas_verbose or needs_build(lib)):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tag = "bc" if bounds_check else "rel"
    os.makedirs(OBJ_DIR, exist_ok=True)
    extra = (["-DMOE_BOUNDS_CHECK"] if bounds_check else []) + (["-Xptxas", "-v"] if ptxas_verbose else [])

    def compile_one(src: str) -> str:
        obj = os.path.join(OBJ_DIR, f"{os.path.splitext(os.path.basename(src))[0]}.{tag}.{os.getpid()}.o")
        subprocess.check_call([nvcc, *COMPILE_FLAGS, *extra, "-c", "-o", obj, src])
        return obj

    srcs = sources()
    with ThreadPoolExecutor(max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(compile_one, srcs))
    tmp = lib + f".tmp{os.getpid()}"
    try:
        subprocess.check_call([nvcc, *LINK_FLAGS, "-o", tmp, *objs])
        os.replace(tmp, lib)
    finally:
        for o in objs:
            if os.path.exists(o):
                os.remove(o)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_verbose="--ptxas-verbose" in sys.argv,
                bounds_check="--bounds-check" in sys.argv))
