"""Build libpa.so in-tree with nvcc for sm_100a (no JIT cache, no torch extension)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libpa.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2",
    "-shared",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _inputs() -> list[str]:
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) +
                              glob.glob(os.path.join(CSRC, "*.h")) +
                              glob.glob(os.path.join(INCLUDE, "*.h")))


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _inputs())


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    return "nvcc"


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    """Compile every .cu under csrc/ into libpa.so (only when sources changed)."""
    if not force and not stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc()] + NVCC_FLAGS + (extra or []) + ["-I", INCLUDE, "-o", tmp] + sources()
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


# Test-only builds of the same sources with extra defines. "waittest": every
# K/V tile wait of the decode kernels reports at once that it ran out of time
# (PA_TEST_TILE_WAIT_EXPIRED), so tests take the timeout path without
# withholding any copy.
VARIANTS = {"waittest": ["-DPA_TEST_TILE_WAIT_EXPIRED"]}


def variant_path(name: str) -> str:
    return os.path.join(PKG, f"libpa_{name}.so")


def build_variant(name: str, force: bool = False, verbose: bool = False) -> str:
    """Compile the test-only library `name` (see VARIANTS) next to libpa.so."""
    out = variant_path(name)
    if not force and os.path.exists(out) and \
            all(os.path.getmtime(f) <= os.path.getmtime(out) for f in _inputs()):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc()] + NVCC_FLAGS + VARIANTS[name] + ["-I", INCLUDE, "-o", tmp] + sources()
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
    print(LIB)
