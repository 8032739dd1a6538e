"""Build libss.so (the sm_100a selective-scan library) in-tree with nvcc.

    python -m selective_state_space_11_b200.build [--verbose]

The library is compiled for sm_100a only (B200); it links the CUDA runtime
statically and exports the C ABI of include/ss.h.
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libss.so")
SOURCES = ["ss_api.cu", "ss_fwd.cu", "ss_bwd.cu", "ss_bwd_ch.cu", "ss_update.cu", "ss_conv.cu", "ss_ssd.cu", "ss_ssd_tc.cu", "ss_ssd_bwd.cu", "ss_ssd_bwd_tc.cu", "ss_shard.cu"]
HEADERS = ["ss_device.cuh", "ss_internal.h", "ss_ssd_bwd.h", "ss_tc.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "ss.h"))
    return any(os.path.getmtime(f) > t for f in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [_nvcc()] + NVCC_FLAGS + (["-Xptxas", "-v"] if verbose else []) + [
        "-shared", "-o", tmp] + [os.path.join(CSRC, f) for f in SOURCES]
    subprocess.check_call(cmd, cwd=CSRC)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/spill report")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force or a.verbose, verbose=a.verbose))
    sys.exit(0)
