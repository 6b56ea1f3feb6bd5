"""Builds the CUDA C-ABI library ``libgdn_b200.so`` in-tree for sm_100a.

    python -m hybrid_linear_attention_step_b200.build [--force] [--verbose]

nvcc cross-compiles without a GPU.  The library links the CUDA runtime
statically, so it loads in any process (torch's own runtime included) and
needs only the driver at run time.
"""
from __future__ import annotations

import argparse
import os
import pathlib
import subprocess

PKG = pathlib.Path(__file__).resolve().parent
ROOT = PKG.parent
SOURCES = [PKG / "csrc" / "gdn_step.cu", PKG / "csrc" / "gdn_prefill_chunked.cu", PKG / "csrc" / "slot_cache.cpp"]
HEADERS = [ROOT / "include" / "gdn_step.h", ROOT / "include" / "gdn_slot_cache.h"]
LIB_PATH = PKG / "libgdn_b200.so"

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-warn-spills",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _stale() -> bool:
    if not LIB_PATH.exists():
        return True
    t = LIB_PATH.stat().st_mtime
    return any(p.stat().st_mtime > t for p in SOURCES + HEADERS + [pathlib.Path(__file__)])


def build(force: bool = False, verbose: bool = False) -> pathlib.Path:
    if not force and not _stale():
        return LIB_PATH
    tmp = LIB_PATH.with_name(f".{LIB_PATH.name}.{os.getpid()}.tmp")
    cmd = [nvcc(), *NVCC_FLAGS, "-I", str(ROOT / "include"), "-o", str(tmp), *map(str, SOURCES)]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose))
