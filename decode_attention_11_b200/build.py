"""Build the tq shared library in-tree for sm_100a (nvcc, no JIT cache).

    python -m decode_attention_11_b200.build [--force] [--debug]

``--debug`` builds ``libtq_b200_debug.so`` as well: the same library with the decode kernel's
device-side bounds checks compiled in (``-DTQ_DEBUG``; a stage's cache rows and ring slot and every
partial slot are checked before use, and a failed check is recorded in the device error word instead
of touching memory).  The package loads it when ``TQ_DEBUG=1`` is set in the environment.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libtq_b200.so")
DEBUG_LIB = os.path.join(HERE, "libtq_b200_debug.so")
DEBUG_SOURCES = ("tq_decode.cu",)  # the sources that hold TQ_DEBUG checks
SOURCES = ["tq_host.cpp", "tq_quantize.cu", "tq_quantize_pipe.cu", "tq_decode.cu"]
HEADERS = [os.path.join(CSRC, "tq_internal.h"), os.path.join(CSRC, "tq_sm100.h"),
           os.path.join(INCLUDE, "tq.h")]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-O2"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + HEADERS + [os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str, obj: str, extra: list, verbose: bool) -> None:
    cmd = [_nvcc()] + NVCC_FLAGS + extra + ["-I", INCLUDE, "-c", os.path.join(CSRC, src), "-o", obj]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)


def _link(objs: list, lib: str) -> None:
    tmp = lib + ".tmp"
    subprocess.run([_nvcc()] + NVCC_FLAGS + ["-shared", "-o", tmp] + objs, check=True)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Build libtq_b200.so (or, with ``debug``, libtq_b200_debug.so, which shares the release
    objects of the sources without checks) and return its path."""
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = {src: os.path.join(objdir, src.rsplit(".", 1)[0] + ".o") for src in SOURCES}
    if force or _stale(LIB):
        for src in SOURCES:
            _compile(src, objs[src], [], verbose)
        _link(list(objs.values()), LIB)
    if not debug:
        return LIB
    if force or _stale(DEBUG_LIB) or os.path.getmtime(LIB) > os.path.getmtime(DEBUG_LIB):
        for src in DEBUG_SOURCES:
            objs[src] = os.path.join(objdir, src.rsplit(".", 1)[0] + "_debug.o")
            _compile(src, objs[src], ["-DTQ_DEBUG"], verbose)
        _link(list(objs.values()), DEBUG_LIB)
    return DEBUG_LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
