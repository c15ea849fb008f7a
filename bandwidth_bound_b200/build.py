"""Build libmk.so (the decode megakernel and its C ABI) in-tree for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmk.so")
SOURCES = ["mk_api.cu", "mk_kernel.cu", "mk_plan.cpp", "kpo.cu"]
HEADERS = ["mk_common.h", "mk_kernel.h", "mk_plan.h"]
PUBLIC_HEADER = os.path.join(os.path.dirname(HERE), "include", "mk.h")


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [PUBLIC_HEADER, __file__]
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force: bool = False, verbose: bool = False, trace_detail: bool = False) -> str:
    """trace_detail: record in-task cycle counts in the per-task timeline (a diagnostic build;
    the stamps cost a few percent of the step)."""
    if not force and not trace_detail and not needs_build():
        return LIB
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared", "-cudart", "static",
           "-o", LIB + ".tmp"] + [os.path.join(CSRC, s) for s in SOURCES]
    if trace_detail:
        cmd.insert(1, "-DMK_TRACE_DETAIL=1")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True, cwd=CSRC)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, trace_detail="--trace-detail" in sys.argv)
    print(LIB)
