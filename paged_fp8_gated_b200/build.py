"""Build libgad_attn.so in-tree with nvcc for sm_100a.

    python -m paged_fp8_gated_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libgad_attn.so")

NVCC_FLAGS = [
    "-O3", "-std=c++17",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo",
    "-Xcompiler", "-fPIC",
    "-shared",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (_sources() + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)])


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(d) > t for d in _deps())


def build(force: bool = False, verbose: bool = False, defines: dict | None = None,
          lib: str = LIB) -> str:
    """Compile the library into `lib` (the package's libgad_attn.so unless a
    variant path is given), with extra -D defines for variant builds."""
    if not force and not stale(lib):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + f".tmp{os.getpid()}"
    dflags = [f"-D{k}={v}" for k, v in sorted((defines or {}).items())]
    cmd = [nvcc, *NVCC_FLAGS, *dflags, "-I", INCLUDE, "-o", tmp, *_sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


# A variant for the tests of the give-up path: every pipeline wait whose phase
# has not completed at its first, non-blocking probe gives up at once (the
# waits before a kernel frees its tensor memory and exits keep their full
# limit).
SHORT_WAIT_LIB = os.path.join(PKG, "libgad_attn_shortwait.so")


def build_short_wait(force: bool = False) -> str:
    return build(force=force, defines={"GAD_TEST_GIVE_UP_AT_FIRST_MISS": "1"}, lib=SHORT_WAIT_LIB)


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
