"""Builds the CUDA library in-tree with nvcc for sm_100a.

    python -m exact_attention_117_b200.build [--debug]  (or __graft_entry__.build())

``--debug`` builds ``libfa_b200_debug.so`` with ``-DFA_DEBUG``: the same
kernels with every TMA coordinate, TMEM column range and directly indexed
global address checked before use (a failed check is reported through the
device error word, see ``fa_check_device_error``).  Point the binding at it
with the ``FA_LIBRARY`` environment variable.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libfa_b200.so")
DEBUG_LIB = os.path.join(PKG, "libfa_b200_debug.so")
SOURCES = ["fa_api.cu"]
HEADERS = ["sm100.cuh", "common.cuh", "fwd.cuh", "bwd.cuh", "bwd_main.cuh", "dq_pass.cuh", "kv_outer.cuh"]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def flags(extra=()):
    return [
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-std=c++17", "-lineinfo",
        "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
        "-shared", "--expt-relaxed-constexpr",
        "-I", os.path.join(ROOT, "include"),
        *extra,
    ]


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "fa.h"))
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def build(force: bool = False, verbose: bool = False, extra=(), debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + ".tmp"
    flag_list = flags(list(extra) + (["-DFA_DEBUG"] if debug else []))
    cmd = [nvcc(), *flag_list, "-o", tmp] + [os.path.join(CSRC, s) for s in SOURCES]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv,
                extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []))
