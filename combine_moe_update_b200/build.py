"""Build libmoe_b200.so (sm_100a) in-tree with nvcc.

    python -m combine_moe_update_b200.build [--force]

The library links the CUDA runtime statically, so it loads on machines
without a GPU driver (every call then returns MOE_ERR_CUDA).  Flags: no
fast-math; quantization relies on IEEE round-to-nearest arithmetic.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(PKG, "_lib")
LIB_PATH = os.path.join(LIB_DIR, "libmoe_b200.so")
# Test-only build: every kernel with a bulk copy can leave one out, so that
# the tests can run the bounded waits' timeout path (never shipped, never
# loaded by the package).
FAULT_LIB_PATH = os.path.join(LIB_DIR, "libmoe_b200_faultinj.so")
PTXAS_LOG = os.path.join(LIB_DIR, "ptxas.log")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "--cudart", "static",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
    "-Xptxas", "-v",
    "-shared",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmoe_b200.so")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def stale(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, fault_injection: bool = False) -> str:
    path = FAULT_LIB_PATH if fault_injection else LIB_PATH
    if not force and not stale(path):
        return path
    os.makedirs(LIB_DIR, exist_ok=True)
    tmp = path + f".tmp{os.getpid()}"
    extra = ["-DMOE_FAULT_INJECTION"] if fault_injection else []
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-o", tmp, os.path.join(CSRC, "moe_b200.cu")]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    log = PTXAS_LOG if not fault_injection else PTXAS_LOG + ".faultinj"
    with open(log, "w") as f:
        f.write(" ".join(cmd) + "\n" + proc.stdout + proc.stderr)
    if proc.returncode != 0:
        sys.stderr.write(proc.stdout + proc.stderr)
        raise RuntimeError(f"nvcc failed ({proc.returncode}); see {log}")
    if verbose:
        sys.stdout.write(proc.stdout + proc.stderr)
    os.replace(tmp, path)
    return path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, fault_injection="--fault-injection" in sys.argv))
