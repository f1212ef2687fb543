"""Build the q4gsw CUDA library in-tree (sm_100a).

``python -m bit_group_quantized_q4gsw_b200.build`` compiles every source under
``csrc/`` into ``libq4gsw.so`` next to this file with nvcc.  The result has no
dependency on torch: it links the CUDA runtime statically and exports only the
C functions declared in ``include/q4gsw.h``.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
LIB_PATH = os.path.join(PKG_DIR, "libq4gsw.so")
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(PKG_DIR, "csrc", "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(PKG_DIR, "csrc", "*.cuh")) + glob.glob(os.path.join(PKG_DIR, "csrc", "*.h"))
                  + glob.glob(os.path.join(ROOT, "include", "*.h")))


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the q4gsw CUDA library cannot be built")


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(f) <= t for f in sources() + headers() + [__file__])


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB_PATH
    cmd = [nvcc_path(), "-std=c++17", "-O3", "-lineinfo", *ARCH_FLAGS, "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include"),
           "-o", LIB_PATH + ".tmp", *sources()]
    if verbose:
        print(" ".join(cmd))
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
