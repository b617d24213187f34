"""Build libqsa.so (the C-ABI CUDA library) in-tree with nvcc for sm_100a.

    python -m top_sparse_attention_index_b200.build_lib [--force] [--verbose-ptxas]

The library links the CUDA runtime statically, so the only run-time dependency is the
NVIDIA driver.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
INCLUDE = ROOT / "include"
LIBRARY = PKG / "libqsa.so"
SOURCES = [CSRC / "qsa_api.cu", CSRC / "qsa_attn.cu", CSRC / "qsa_noalloc.cu", CSRC / "qsa_probe.cu",
           CSRC / "qsa_probe_mma.cu", CSRC / "qsa_peer.cu"]
DEPENDS = SOURCES + [CSRC / "qsa_internal.h", CSRC / "qsa_ptx.cuh", INCLUDE / "qsa.h",
                     INCLUDE / "qsa_probe.h", INCLUDE / "qsa_peer.h"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-Xcompiler", "-Wall",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and Path(cand).exists():
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libqsa.so")


def build(force: bool = False, verbose_ptxas: bool = False, output: Path = LIBRARY) -> Path:
    output = Path(output)
    if (not force and output.exists()
            and output.stat().st_mtime >= max(p.stat().st_mtime for p in DEPENDS)):
        return output
    cmd = [nvcc(), *NVCC_FLAGS, "-I", str(INCLUDE), "-I", str(CSRC)]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += [str(s) for s in SOURCES] + ["-o", str(output)]
    subprocess.run(cmd, check=True)
    return output


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv))
