"""The tensor-core kernel's work split, checked on the host.

tests/segwalk_check.cu includes the kernel header and compiles SegWalk and
split_owners for the host with nvcc (no GPU needed); the program enumerates
tile counts, chunk counts and grid sizes and checks that every unit is walked
once, that CTAs differ by at most one unit, and that each split tile's owner
range is exactly its set of contributors.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.mark.skipif(not (os.path.exists(NVCC) or shutil.which("nvcc")), reason="nvcc not available")
def test_segwalk_covers_balances_and_owns(tmp_path):
    exe = tmp_path / "segwalk_check"
    nvcc = NVCC if os.path.exists(NVCC) else shutil.which("nvcc")
    subprocess.run([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "sparse_bit_matmul_b200", "csrc"),
                    os.path.join(HERE, "segwalk_check.cu"), "-o", str(exe)], check=True,
                   capture_output=True, text=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stdout + res.stderr
    assert res.stdout.startswith("ok")
