"""The C ABI from a C program: tests/c/qsa_c_caller.c links libqsa.so (and, for the check
only, the CPU oracle) with no Python in between.  Compiling it needs no GPU; running it
does."""
from __future__ import annotations

import shutil
import subprocess
from pathlib import Path

import pytest

import oracle
from top_sparse_attention_index_b200 import build_lib

ROOT = Path(__file__).resolve().parent.parent
SOURCE = ROOT / "tests" / "c" / "qsa_c_caller.c"


def _cuda_home() -> Path:
    return Path(build_lib.nvcc()).resolve().parent.parent


def _build(tmp: Path) -> Path:
    lib = build_lib.build()
    orc = oracle.build()
    cuda = _cuda_home()
    exe = tmp / "qsa_c_caller"
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-I", str(ROOT / "include"),
           "-I", str(cuda / "include"), str(SOURCE), "-o", str(exe),
           str(lib), str(orc), "-L", str(cuda / "lib64"), "-lcudart", "-lm",
           f"-Wl,-rpath,{lib.parent}:{orc.parent}:{cuda / 'lib64'}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc is needed to build the C caller")
def test_c_caller_builds(tmp_path):
    assert _build(tmp_path).exists()


@pytest.mark.gpu
def test_c_caller_matches_oracle(cuda_device, tmp_path):
    exe = _build(tmp_path)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    print(out.stdout)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip().endswith("OK")
