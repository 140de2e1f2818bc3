"""Build the in-tree CUDA library ``libhvattn.so`` for sm_100a with nvcc.

The library is built in the package directory (not installed anywhere else)
so that it travels with the source tree. ``python -m
joint_full_attention_b200.build`` rebuilds it when a source is newer.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
SOURCES = [PKG / "csrc" / "hv_attn.cu"]
HEADERS = [PKG / "csrc" / "sm100_ptx.cuh", ROOT / "include" / "hv_attn.h"]
LIB = PKG / "libhvattn.so"

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2", "-shared",
    "-Xptxas", "-v",
]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and Path(cand).exists():
            return cand
    raise RuntimeError("nvcc not found: cannot build the sm_100a library")


def is_stale() -> bool:
    if not LIB.exists():
        return True
    built = LIB.stat().st_mtime
    return any(src.stat().st_mtime > built for src in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False) -> Path:
    """Compile ``libhvattn.so`` if missing or older than its sources."""
    if not force and not is_stale():
        return LIB
    tmp = LIB.with_suffix(".so.tmp")
    cmd = [nvcc_path(), *NVCC_FLAGS, "-I", str(ROOT / "include"), "-o", str(tmp), *map(str, SOURCES)]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        raise RuntimeError(f"nvcc failed ({proc.returncode}):\n{proc.stdout}\n{proc.stderr}")
    if verbose:
        sys.stderr.write(proc.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
