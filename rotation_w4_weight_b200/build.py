"""Builds the CUDA library in-tree: rotation_w4_weight_b200/libparo_b200.so (sm_100a).

The whole library is one translation unit (csrc/paro_abi.cu includes the
kernel headers), compiled with nvcc for sm_100a only and linked against the
static CUDA runtime.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "paro_abi.cu")
OUT = os.path.join(PKG, "libparo_b200.so")
HEADERS = [os.path.join(PKG, "csrc", f) for f in sorted(os.listdir(os.path.join(PKG, "csrc")))]
HEADERS.append(os.path.join(ROOT, "include", "paro.h"))

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v",
]


def nvcc_path() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build the library")
    return cand


def needs_build() -> bool:
    if not os.path.exists(OUT):
        return True
    t = os.path.getmtime(OUT)
    return any(os.path.getmtime(h) > t for h in HEADERS if os.path.exists(h))


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if any source is newer than the .so.  Returns its path."""
    if not force and not needs_build():
        return OUT
    cmd = [nvcc_path(), *NVCC_FLAGS, "-o", OUT + ".tmp", SRC]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stdout.write(res.stderr)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
