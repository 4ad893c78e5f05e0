"""CPU comparison kernel: the Sherry page's x86 table-lookup scheme
(``sherry_cpu_lut.c``; Sherry page, pnsm.cn/news/1195499, sec. 2.2 steps 1-4
and sec. 5.1: a 16-entry table per 4-element activation segment, vpshufb
lookups, sign application, integer sums, one float scaling).

It is the stronger timed CPU baseline of bench.py.  It is neither the oracle
nor part of the GPU library: nothing under sparse_bit_matmul_b200/ imports
it, and it shares no code with either.  Only tests/ and bench.py load it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsherry_cpu_lut.so")
_lib = None


class LutError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "sherry_cpu_lut.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", _SO, src])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        i64, vp = ctypes.c_int64, ctypes.c_void_p
        L.lut_prepared_bytes.argtypes = [i64, i64]
        L.lut_prepared_bytes.restype = i64
        L.lut_prepare.argtypes = [vp, i64, i64, vp]
        L.lut_gemm.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp, ctypes.c_int]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def has_avx2() -> bool:
    return bool(_load().lut_has_avx2())


def num_threads() -> int:
    return int(_load().lut_num_threads())


def prepare(codes: np.ndarray, K: int) -> np.ndarray:
    """Canonical codes [N][5K/32] -> index bytes [row block][group][32]."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N = codes.shape[0]
    out = np.empty(int(_load().lut_prepared_bytes(N, K)), dtype=np.uint8)
    rc = _load().lut_prepare(_p(codes), N, K, _p(out))
    if rc:
        raise LutError(f"lut_prepare: status {rc}")
    return out


def gemm(q: np.ndarray, s: np.ndarray, prepared: np.ndarray, alpha: np.ndarray, N: int, K: int,
         force_scalar: bool = False, want_acc: bool = True):
    """(y fp32 [M][N], acc int32 [M][N] or None) from int8 q [M][K] and scales s [M]."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    s = np.ascontiguousarray(s, dtype=np.float32)
    alpha = np.ascontiguousarray(alpha, dtype=np.float32)
    M = q.shape[0]
    y = np.empty((M, N), dtype=np.float32)
    acc = np.empty((M, N), dtype=np.int32) if want_acc else None
    rc = _load().lut_gemm(_p(q), _p(s), _p(prepared), _p(alpha), M, N, K, _p(y),
                          _p(acc) if acc is not None else None, int(force_scalar))
    if rc:
        raise LutError(f"lut_gemm: status {rc}")
    return y, acc
