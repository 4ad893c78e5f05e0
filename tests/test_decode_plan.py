"""The decode kernel's work split and shared-memory indexing, checked on the host.

tests/decode_plan_check.cu includes the kernel header and compiles decode::plan
and the kernel's index expressions for the host with nvcc (no GPU needed); the
program enumerates token counts, shapes and SM counts and checks that row
ranges tile N, that every (row, K chunk) pair is walked by one thread, and that
every shared-memory and weight index stays inside its buffer.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.mark.skipif(not (os.path.exists(NVCC) or shutil.which("nvcc")), reason="nvcc not available")
def test_decode_plan_tiles_and_stays_in_bounds(tmp_path):
    exe = tmp_path / "decode_plan_check"
    nvcc = NVCC if os.path.exists(NVCC) else shutil.which("nvcc")
    subprocess.run([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "sparse_bit_matmul_b200", "csrc"),
                    os.path.join(HERE, "decode_plan_check.cu"), "-o", str(exe)], check=True,
                   capture_output=True, text=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
    assert res.stdout.startswith("ok")
