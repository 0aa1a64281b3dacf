"""Build the CUDA shared library (sm_100a) in-tree with nvcc.

The library is one translation unit (csrc/moe_api.cu includes the kernel headers) and
exports the C ABI declared in include/moe.h.
"""
from __future__ import annotations

import os
import shutil
import subprocess
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
INCLUDE = ROOT / "include"
LIB_PATH = PKG / "libmoe_b200.so"

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xcompiler", "-fvisibility=hidden",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and Path(cand).exists():
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(CSRC.glob("*.cu")) + sorted(CSRC.glob("*.cuh")) + [INCLUDE / "moe.h"]


def needs_build(out: Path = LIB_PATH) -> bool:
    if not out.exists():
        return True
    t = out.stat().st_mtime
    return any(s.stat().st_mtime > t for s in _sources())


def build_library(force: bool = False, out: Path = LIB_PATH, extra_flags=()) -> Path:
    """Compile csrc/moe_api.cu into ``out`` (default: the in-tree libmoe_b200.so)."""
    out = Path(out)
    if not force and not needs_build(out):
        return out
    tmp = out.with_name(out.name + f".tmp{os.getpid()}")
    cmd = [_nvcc(), *NVCC_FLAGS, *extra_flags, "-I", str(INCLUDE), "-o", str(tmp),
           str(CSRC / "moe_api.cu")]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build_library(force=True))
