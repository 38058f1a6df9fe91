"""Builds libcmr.so, the C-ABI library, in-tree with nvcc for sm_100a (B200),
and libcmr_probe.so, the benchmark's copy-pattern ceiling probe.

    python -m vlm_decoder_positional_b200.build [--force] [--verbose-ptxas]

The CUDA runtime is linked statically, so the libraries need only the NVIDIA
driver at run time.  Only the symbols declared in include/cmr.h are exported
from libcmr.so.
"""
import argparse
import glob
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
INCLUDE = os.path.join(ROOT, "include")
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libcmr.so")
PROBE_DIR = os.path.join(PKG, "probe")
PROBE_LIB = os.path.join(PKG, "libcmr_probe.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden,-O2,-Wall",
    "-cudart", "static",
    "--shared",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def probe_sources():
    return sorted(glob.glob(os.path.join(PROBE_DIR, "*.cu")))


def _stale(lib, srcs) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = srcs + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(INCLUDE, "cmr.h"),
                                                           os.path.abspath(__file__)]
    return any(os.path.getmtime(p) > t for p in deps)


def _nvcc(lib, srcs, verbose_ptxas):
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = [NVCC] + NVCC_FLAGS + (["-Xptxas", "-v"] if verbose_ptxas else []) + [
        "-I", INCLUDE, "-o", tmp] + srcs
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    """Builds libcmr.so (and the probe library) when missing or older than
    their sources; returns the path of libcmr.so."""
    if force or _stale(LIB, sources()):
        _nvcc(LIB, sources(), verbose_ptxas)
    if force or _stale(PROBE_LIB, probe_sources()):
        _nvcc(PROBE_LIB, probe_sources(), verbose_ptxas)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force or a.verbose_ptxas, verbose_ptxas=a.verbose_ptxas))
