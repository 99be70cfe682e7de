"""Build the sm_100a shared library ``libmoe_b200.so`` in-tree with nvcc.

Usage: ``python -m sparse_moe_layer_05_b200.build`` (or ``build()``).
The library is written next to this file so that it travels with the source
tree; it links the CUDA runtime statically and needs no torch headers.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmoe_b200.so")
SOURCES = ["moe_abi.cu", "moe_routing.cu", "moe_router_tc.cu", "moe_grouped_gemm.cu",
           "moe_mx_gemm.cu", "moe_mx_pair.cu", "moe_noalloc.cu"]
HEADERS = ["moe_ptx.cuh", "moe_internal.h", "moe_topk.cuh", "moe_perm_small.cuh"]
# the tensor-core rate probe: measurement tooling, a library of its own
PROBE_LIB = os.path.join(PKG, "libmoe_b200_probe.so")
PROBE_SOURCES = ["moe_probe.cu"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(lib: str, sources, headers) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in list(sources) + list(headers)]
    deps += [os.path.join(ROOT, "include", h) for h in ("moe_b200.h", "moe_b200_probe.h")]
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(p) > t for p in deps)


def _nvcc(lib: str, sources, verbose: bool, extra) -> None:
    tmp = lib + ".tmp"
    cmd = [nvcc_path(), *NVCC_FLAGS, *extra, "-I", os.path.join(ROOT, "include"),
           "-o", tmp, *[os.path.join(CSRC, f) for f in sources]]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose and res.stderr:
        print(res.stderr, file=sys.stderr)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Build the layer's library and the probe library (each only when stale)."""
    if force or _stale(LIB, SOURCES, HEADERS):
        _nvcc(LIB, SOURCES, verbose, extra)
    if force or _stale(PROBE_LIB, PROBE_SOURCES, ["moe_ptx.cuh"]):
        _nvcc(PROBE_LIB, PROBE_SOURCES, verbose, extra)
    return LIB


if __name__ == "__main__":
    force = "--force" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []
    print(build(force=force, verbose=True, extra=extra))
