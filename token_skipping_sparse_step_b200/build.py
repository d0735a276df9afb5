"""Build the CUDA library ``libesd.so`` in-tree (sm_100a only).

    python token_skipping_sparse_step_b200/build.py

nvcc cross-compiles without a GPU. The CUDA runtime is linked statically and
the driver entry point for TMA descriptors is resolved at run time, so the
library loads on a machine without a driver (its entry points then return
ESD_ERR_CUDA / ESD_ERR_UNSUPPORTED).
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libesd.so")
PROBE_SRC = os.path.join(CSRC, "stream_probe.cu")
PROBE_LIB = os.path.join(PKG, "libstream_probe.so")
SYNTH_SRC = os.path.join(ROOT, "synth", "csrc", "synth.cu")
SYNTH_LIB = os.path.join(ROOT, "synth", "libsynth.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2,-Wall,-Wno-unused-function",
    "-Xptxas", "-warn-spills,-warn-lmem-usage",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def sources():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))
            if f.endswith((".cu", ".cuh")) and f != "stream_probe.cu"]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + [os.path.join(INCLUDE, "esd.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(verbose: bool = False, extra=()) -> str:
    cmd = [_nvcc(), *NVCC_FLAGS, *extra, "-shared", "-I", INCLUDE, "-I", CSRC,
           os.path.join(CSRC, "esd_api.cu"), "-o", LIB]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    return LIB


def build_synth(verbose: bool = False) -> str:
    """The seeded input generator's CUDA twin (not part of the method)."""
    cmd = [_nvcc(), *NVCC_FLAGS, "-shared", SYNTH_SRC, "-o", SYNTH_LIB]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    return SYNTH_LIB


def build_stream_probe(verbose: bool = False) -> str:
    """The HBM streaming probe behind the roofline notes (bench.py --stream-probe)."""
    cmd = [_nvcc(), *NVCC_FLAGS, "-shared", PROBE_SRC, "-o", PROBE_LIB]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    return PROBE_LIB


def build_all(verbose: bool = False):
    build(verbose=verbose)
    build_synth(verbose=verbose)
    build_stream_probe(verbose=verbose)


if __name__ == "__main__":
    build(verbose=True, extra=sys.argv[1:])
    build_synth(verbose=True)
    build_stream_probe(verbose=True)
