"""Build libefla.so (all CUDA sources of csrc/) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libefla.so")
# the checked build: every direct global access and computed shared-memory store of the
# tensor-core forward is tested against its buffer (EFLA_CHECKED=1 in csrc/efla_common.cuh)
LIB_CHECKED = os.path.join(PKG, "libefla_checked.so")
INCLUDE = os.path.join(os.path.dirname(PKG), "include")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(out: str) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps += glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra=(), checked: bool = False) -> str:
    out = LIB_CHECKED if checked else LIB
    if not force and not _stale(out):
        return out
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = out + f".tmp{os.getpid()}"
    flags = list(extra) + (["-DEFLA_CHECKED=1"] if checked else [])
    cmd = [nvcc, *NVCC_FLAGS, *flags, "-I", INCLUDE, "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, checked="--checked" in sys.argv))
