"""Build ``libkda_decode.so`` in-tree with nvcc for sm_100a.

    python -m linear_attention_recurrent_decode_b200.build [--force] [-v]

The library is the C ABI declared in ``include/kda_decode.h`` and
``include/kda_prefill.h``: the CUDA translation units under ``csrc/`` (one per
decode key size, the decode and prefill entry points) are compiled in
parallel for ``sm_100a`` only and linked into one shared object, with the CUDA
runtime linked statically so it loads on its own (no torch, no JIT cache).
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libkda_decode.so")
OBJDIR = os.path.join(ROOT, "_build")
SOURCES = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))
DEPENDS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + [
    os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in DEPENDS)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if it is missing or older than its sources."""
    if not force and not stale():
        return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    tag = f".{os.getpid()}"
    objs = [os.path.join(OBJDIR, os.path.basename(src)[:-3] + tag + ".o") for src in SOURCES]

    def compile_one(src_obj):
        src, obj = src_obj
        cmd = [_nvcc(), *NVCC_FLAGS, "-c", "-I", INCLUDE, "-I", CSRC, "-o", obj, src]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)

    try:
        with ThreadPoolExecutor(max_workers=max(1, min(len(SOURCES), os.cpu_count() or 1))) as ex:
            list(ex.map(compile_one, zip(SOURCES, objs)))
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call([_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                               "-Xcompiler", "-fPIC", "-o", tmp, *objs])
        os.replace(tmp, LIB)
    finally:
        for o in objs:
            if os.path.exists(o):
                os.remove(o)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
