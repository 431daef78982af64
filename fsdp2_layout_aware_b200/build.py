"""Build libtide.so in-tree with nvcc for sm_100a.

    python -m fsdp2_layout_aware_b200.build [-v]

Objects go to fsdp2_layout_aware_b200/_build/, the library to
fsdp2_layout_aware_b200/libtide.so.  The CUDA runtime is linked statically so
the library does not depend on which libcudart the host process loaded.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libtide.so")
INCLUDE = os.path.join(ROOT, "include")

SOURCES = ["plan.cpp", "api.cpp", "ce.cpp", "rs_reduce.cu", "rs_reduce_tma.cu", "ag_place.cu",
           "rs_reduce_noalloc.cu", "ipc.cpp", "flags.cu", "f32_grads.cu"]
HEADERS = ["tide_internal.h", "device_common.cuh", "reduce_ranks.cuh", "tma.cuh"]

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "--fmad=false", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall", "-Xcompiler", "-fvisibility=hidden",
              "-I", INCLUDE, "-I", CSRC]


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, ptxas_verbose: bool = False, force: bool = False,
          defines=(), build_dir: str = BUILD, lib_path: str = LIB, src_dir: str = CSRC,
          include_dir: str = INCLUDE) -> str:
    """Compile (incrementally) and link; `defines` are extra -D tuning macros."""
    os.makedirs(build_dir, exist_ok=True)
    headers = [os.path.join(src_dir, h) for h in HEADERS] + [os.path.join(include_dir, "tide.h")]
    flags = [f for f in NVCC_FLAGS]
    flags[flags.index(INCLUDE)] = include_dir
    flags[flags.index(CSRC)] = src_dir
    objs = []
    for src in SOURCES:
        path = os.path.join(src_dir, src)
        obj = os.path.join(build_dir, src + ".o")
        objs.append(obj)
        if not force and not _stale(obj, [path] + headers + [__file__]):
            continue
        cmd = ["nvcc", *flags, *[f"-D{d}" for d in defines], "-c", path, "-o", obj]
        if ptxas_verbose and src.endswith(".cu"):
            cmd[1:1] = ["-Xptxas", "-v"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    if force or _stale(lib_path, objs):
        cmd = ["nvcc", "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-cudart", "static",
               "-o", lib_path, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return lib_path


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, ptxas_verbose="--ptxas" in sys.argv, force="-f" in sys.argv)
