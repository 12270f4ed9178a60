"""Builds libqlora.so in-tree with nvcc for sm_100a (B200).

    python -m qlora_parameter_efficient_b200.build            # release: libqlora.so
    python -m qlora_parameter_efficient_b200.build --debug    # libqlora_debug.so, QLORA_DEBUG=1

The debug library checks the kernels' index invariants on the device (a failed check is
reported as QLORA_ERR_DEVICE by qlora_get_device_error); load it with QLORA_LIB=<path>.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libqlora.so")
DEBUG_LIB = os.path.join(HERE, "libqlora_debug.so")
SOURCES = ["qlora_api.cu", "noalloc.cu"]
DEPS = sorted(f for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh")))
HEADER = os.path.join(os.path.dirname(HERE), "include", "qlora.h")

NVCC_FLAGS = [
    "-std=c++17", "-O3", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-shared", "-Xcompiler", "-fPIC",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, d) for d in DEPS] + [HEADER]
    return all(os.path.getmtime(d) <= t for d in deps if os.path.exists(d))


def build_library(force: bool = False, verbose: bool = False, debug: bool = False, out: str = None) -> str:
    lib = out or (DEBUG_LIB if debug else LIB)
    if not force and up_to_date(lib):
        return lib
    flags = NVCC_FLAGS + (["-DQLORA_DEBUG=1"] if debug else [])
    cmd = [nvcc(), *flags, "-o", lib + ".tmp", *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libqlora.so")
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build_library(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
