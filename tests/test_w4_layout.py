"""The W4A8 kernel-native layout, checked on the host.

tests/w4_layout_check.cpp builds native words with the library's own
sherry_w4_native_word (the body of the repack kernel) and decodes them the
way the tensor-core kernel's decoder warps do: every int8 must be 16 w (the
SINT4toS8 shift of the OdysseyLLM review page, sec. 3.2 / 5.2) at its TMEM
column, with zeros past N and K.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def test_w4_native_layout_decodes_to_16w(tmp_path):
    exe = tmp_path / "w4_layout_check"
    subprocess.run(["g++", "-std=c++17", "-O2", "-I", os.path.join(ROOT, "sparse_bit_matmul_b200", "csrc"),
                    os.path.join(HERE, "w4_layout_check.cpp"), "-o", str(exe)], check=True,
                   capture_output=True, text=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stdout + res.stderr
    assert res.stdout.startswith("ok")
