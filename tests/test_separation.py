"""The product, the oracle and the CPU comparison kernel stay apart.

- Nothing under sparse_bit_matmul_b200/ imports or includes oracle/ or
  cpu_lut/, and importing the package loads neither module.
- oracle/ and cpu_lut/ C sources include system headers only: no header of
  the CUDA library (sparse_bit_matmul_b200/csrc, include/).
- synth/ (the seeded generators both sides share) includes system headers
  only as well.
"""
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _files(sub, exts):
    for dp, _, fs in os.walk(os.path.join(ROOT, sub)):
        for f in fs:
            if f.endswith(exts):
                yield os.path.join(dp, f)


def test_product_never_imports_oracle_or_cpu_lut():
    py_imp = re.compile(r"^\s*(import|from)\s+(oracle|cpu_lut)\b", re.M)
    c_inc = re.compile(r'^\s*#\s*include\s*[<"][^>"]*(oracle|cpu_lut)', re.M)
    for f in _files("sparse_bit_matmul_b200", (".py", ".cu", ".cuh", ".h", ".cpp")):
        text = open(f, encoding="utf-8").read()
        assert not py_imp.search(text), f"{f} imports the oracle or the CPU comparison kernel"
        assert not c_inc.search(text), f"{f} includes the oracle or the CPU comparison kernel"


def test_importing_the_product_loads_neither():
    code = ("import sys; sys.path.insert(0, %r); import sparse_bit_matmul_b200 as s; "
            "bad = [m for m in ('oracle', 'cpu_lut') if m in sys.modules]; "
            "print(bad); sys.exit(1 if bad else 0)") % ROOT
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr


def test_reference_side_c_sources_include_system_headers_only():
    inc = re.compile(r'^\s*#\s*include\s*(.+)$', re.M)
    for sub in ("oracle", "cpu_lut", "synth"):
        for f in _files(sub, (".c", ".h")):
            for target in inc.findall(open(f, encoding="utf-8").read()):
                assert target.strip().startswith("<"), f"{f} includes {target.strip()}"
