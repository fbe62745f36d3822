"""Build libattn.so in-tree with nvcc for sm_100a.

    python bwd_causal_sdpa_b200/build.py [--force] [--debug]

--debug builds libattn_debug.so, the watchdog test library (debug hooks on,
bounded waits cut to ~10 ms); the product is libattn.so.

The library is one translation unit (csrc/attn_api.cu, which includes the
kernel headers); cudart is linked statically, and the CUDA driver entry point
the TMA descriptors need is fetched at run time, so the .so depends on
nothing beyond the driver of the machine it runs on.
"""

from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libattn.so")
INCLUDE = os.path.join(ROOT, "include")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _sources():
    out = []
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh")):
            out.append(os.path.join(CSRC, name))
    out.append(os.path.join(INCLUDE, "attn.h"))
    return out


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in _sources())


def up_to_date_at(lib: str) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in _sources())


def _compile(lib: str, flags, verbose: bool) -> str:
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *NVCC_FLAGS, *flags, "-I", INCLUDE, "-I", CSRC,
           os.path.join(CSRC, "attn_api.cu"), "-o", lib + ".tmp"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


def build(force: bool = False, verbose: bool = False, extra_flags=None) -> str:
    if not force and up_to_date():
        return LIB
    return _compile(LIB, list(extra_flags or []), verbose)


# The test library: the same sources with the debug hooks compiled in
# (attn_debug_withhold works), the bounded waits cut to 2e7 cycles (~10 ms),
# and the backward's dQ formed by the other of its two routes than the
# product library's, so that the GPU tests cover both.
LIB_DEBUG = os.path.join(PKG, "libattn_debug.so")
DEBUG_FLAGS = ["-DATTN_DEBUG_HOOKS", "-DATTN_WAIT_LIMIT_CYCLES=20000000LL", "-DATTN_DQ_ROUTE_SWAPPED"]


def build_debug(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date_at(LIB_DEBUG):
        return LIB_DEBUG
    return _compile(LIB_DEBUG, DEBUG_FLAGS, verbose)


if __name__ == "__main__":
    args = sys.argv[1:]
    extra = [a for a in args if a.startswith("-X") or a.startswith("--ptxas")]
    if "--debug" in args:
        print(build_debug(force="--force" in args, verbose=True))
    else:
        print(build(force="--force" in args, verbose=True, extra_flags=extra))
