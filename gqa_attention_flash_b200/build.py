"""Build ``libgqa_attn.so`` in-tree with nvcc for sm_100a.

Usage: ``python -m gqa_attention_flash_b200.build`` (or ``build()`` from Python).
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
LIBRARY = os.path.join(PKG, "libgqa_attn.so")
# Checked build: every TMA coordinate and global index is range-checked in the
# kernels (a violation sets ATTN_ERR_DEVICE_BOUNDS and the kernel gives up).
DEBUG_LIBRARY = os.path.join(PKG, "libgqa_attn_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def up_to_date(output: str = LIBRARY) -> bool:
    if not os.path.exists(output):
        return False
    t = os.path.getmtime(output)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) \
        + glob.glob(os.path.join(INCLUDE, "*.h"))
    return all(os.path.getmtime(d) <= t for d in deps)


def build(output: str = LIBRARY, verbose_ptxas: bool = False, force: bool = False,
          debug: bool = False) -> str:
    """Compile every .cu under csrc/ into one shared library (sm_100a); with
    debug=True the checked build (-DGQA_ATTN_DEBUG) into libgqa_attn_debug.so."""
    if debug and output == LIBRARY:
        output = DEBUG_LIBRARY
    if not force and up_to_date(output):
        return output
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC, *sources(), "-o", output]
    if debug:
        cmd.insert(1, "-DGQA_ATTN_DEBUG")
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    return output


if __name__ == "__main__":
    debug = "--debug" in sys.argv
    print(build(verbose_ptxas="-v" in sys.argv, force=True, debug=debug))
