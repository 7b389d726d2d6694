"""Build libfa_hybrid.so in-tree with nvcc for sm_100a (no GPU needed), and
its debug twin libfa_hybrid_debug.so (-DFA_DEBUG=1: each direct global store
of an output is bounds-checked against its tensor and reported in the device
status word instead of being made out of range).

Usage: python -m block_sparse_attention_layerrouter_b200.build [--force] [--debug]
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfa_hybrid.so")
LIB_DEBUG = os.path.join(HERE, "libfa_hybrid_debug.so")
SOURCES = ["fa_api.cu", "fa_router.cu", "fa_index.cu", "fa_prefill.cu", "fa_decode.cu",
           "fa_noalloc.cu", "fa_backward.cu"]
HEADERS = ["fa_common.cuh", "fa_internal.h", os.path.join("..", "..", "include", "fa_hybrid.h")]
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr", "-Xptxas", "-v",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [__file__]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    build_dir = os.path.join(HERE, "_build_debug" if debug else "_build")
    os.makedirs(build_dir, exist_ok=True)
    flags = NVCC_FLAGS + (["-DFA_DEBUG=1"] if debug else [])
    objs, procs = [], []
    for src in SOURCES:                      # the sources compile in parallel
        obj = os.path.join(build_dir, src.replace(".cu", ".o"))
        cmd = [_nvcc(), *flags, "-c", os.path.join(CSRC, src), "-o", obj]
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                            stderr=subprocess.STDOUT, text=True)))
        objs.append(obj)
    for src, proc in procs:
        out, _ = proc.communicate()
        if verbose or proc.returncode != 0:
            sys.stderr.write(out)
        if proc.returncode != 0:
            raise RuntimeError("nvcc failed on %s" % src)
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs,
           "-Xcompiler", "-fPIC"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("link failed")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                debug="--debug" in sys.argv))
