"""Source guards: forms the library must never contain.

- No bulk or tensor copy with cluster multicast anywhere in the sources: a
  multicast load whose source could be another GPU's memory is not to be
  built, and the library runs on several GPUs (one process per GPU).
- No deliberate trap in device code: failures are reported through the
  device status word, never by stopping the GPU.
"""
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SOURCE_DIRS = ["sparse_bit_matmul_b200", "include", "oracle", "cpu_lut", "synth"]
EXTS = (".cu", ".cuh", ".h", ".hpp", ".c", ".cpp", ".py")


def _sources():
    for d in SOURCE_DIRS:
        for base, _, files in os.walk(os.path.join(ROOT, d)):
            for f in files:
                if f.endswith(EXTS):
                    yield os.path.join(base, f)
    yield os.path.join(ROOT, "bench.py")
    yield os.path.join(ROOT, "__graft_entry__.py")


def test_no_cluster_multicast_copies():
    pattern = re.compile(r"\.multi" + r"cast::" + r"cluster")
    hits = []
    for path in _sources():
        with open(path, encoding="utf-8", errors="replace") as fh:
            for n, line in enumerate(fh, 1):
                if pattern.search(line):
                    hits.append(f"{os.path.relpath(path, ROOT)}:{n}")
    assert not hits, hits


def test_no_device_traps():
    pattern = re.compile(r"__tr" + r"ap\s*\(|\btr" + r"ap\s*;")
    hits = []
    for path in _sources():
        if not path.endswith((".cu", ".cuh")):
            continue
        with open(path, encoding="utf-8", errors="replace") as fh:
            for n, line in enumerate(fh, 1):
                if pattern.search(line):
                    hits.append(f"{os.path.relpath(path, ROOT)}:{n}")
    assert not hits, hits
