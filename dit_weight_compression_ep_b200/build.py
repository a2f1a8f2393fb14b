"""Build libentropack.so in-tree: the CUDA decoder (sm_100a) and the C++ packer; and
libep_probe.so, the latency probe behind `bench.py --latency` (not part of the codec).

    python -m dit_weight_compression_ep_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
SO = os.path.join(HERE, "libentropack.so")
PROBE_SO = os.path.join(HERE, "libep_probe.so")
PROBE_SRC = os.path.join(CSRC, "latency_probe.cu")
BUILD = os.path.join(ROOT, "_build")

CU_SOURCES = ["decode.cu", "encode_gpu.cu"]
# the GPU encoder rounds every product and sum as the CPU packer does: no multiply-add contraction
CU_FLAGS = {"encode_gpu.cu": ["-fmad=false", "-Xcompiler", "-ffp-contract=off"]}
CPP_SOURCES = ["encode.cpp"]
HEADERS = ["ep_format.h", "encode_host.h"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _sources():
    out = [os.path.join(CSRC, s) for s in CU_SOURCES + CPP_SOURCES + HEADERS]
    out.append(os.path.join(INCLUDE, "entropack.h"))
    return [s for s in out if os.path.exists(s)]


def _stale() -> bool:
    if not os.path.exists(SO):
        return True
    t = os.path.getmtime(SO)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return SO
    os.makedirs(BUILD, exist_ok=True)
    objs = []
    for src in CU_SOURCES:
        obj = os.path.join(BUILD, src + ".o")
        cmd = [NVCC, *ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
               *CU_FLAGS.get(src, []), "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.check_call(cmd)
        objs.append(obj)
    for src in CPP_SOURCES:
        path = os.path.join(CSRC, src)
        if not os.path.exists(path):
            continue
        obj = os.path.join(BUILD, src + ".o")
        cmd = ["g++", "-std=c++17", "-O2", "-fPIC", "-ffp-contract=off", "-fno-fast-math", "-pthread", "-Wall",
               "-I", INCLUDE, "-I", CSRC, "-c", path, "-o", obj]
        subprocess.check_call(cmd)
        objs.append(obj)
    tmp = SO + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs, "-lpthread"])
    os.replace(tmp, SO)
    build_probe(force)
    return SO


def build_probe(force: bool = False) -> str:
    """The latency probe as its own small library."""
    if force or not os.path.exists(PROBE_SO) or os.path.getmtime(PROBE_SO) < os.path.getmtime(PROBE_SRC):
        tmp = PROBE_SO + f".tmp{os.getpid()}"
        subprocess.check_call([NVCC, *ARCH, "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", PROBE_SRC,
                               "-o", tmp])
        os.replace(tmp, PROBE_SO)
    return PROBE_SO


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(SO)
