"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

This module holds none of the method's arithmetic: it only draws fp32 weights
and activations with the distributions of the Sherry workloads (weights
~N(0, 0.02), activations ~N(0, 1), the heavy-tailed stress case with 1% +-5.0
weight spikes and 1% x20 activation outlier channels).  The generator is
counter based (splitmix64 + Box-Muller, see ``synth.c``), so element ``i`` of
a tensor depends only on its seed and ``i``; any subset of rows can be
regenerated exactly.

Seeds: ``seed(config c, copy r, tensor t) = c * 2**20 + r * 2**4 + t`` with
``t`` = 0 weights, 1 activations, 2 weight spikes, 3 outlier channels.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_lib = None

T_W, T_X, T_SPIKE, T_OUTLIER = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile ``synth.c`` into ``libsynth.so`` next to it."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
             "-o", _SO, src, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        u64, i64, f64 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double
        fp = ctypes.POINTER(ctypes.c_float)
        lib.synth_normal.argtypes = [u64, u64, i64, f64, fp]
        lib.synth_bits.argtypes = [u64, u64, i64, ctypes.POINTER(ctypes.c_uint64)]
        lib.synth_spikes.argtypes = [u64, u64, i64, f64, ctypes.c_float, fp]
        _lib = lib
    return _lib


def seed_of(config: int, copy: int, tensor: int) -> int:
    return config * (1 << 20) + copy * (1 << 4) + tensor


def _fptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def normal(seed: int, n: int, sigma: float, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    _load().synth_normal(seed, offset, n, sigma, _fptr(out))
    return out


def bits(seed: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _load().synth_bits(seed, offset, n, out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64)))
    return out


def weights(config: int, copy: int, N: int, K: int, rows=None, *, sigma: float = 0.02,
            spike_p: float = 0.0, spike_mag: float = 5.0) -> np.ndarray:
    """fp32 W[N][K] (or only ``rows`` of it), row-major, element n*K+k."""
    rows = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), K), dtype=np.float32)
    lib = _load()
    s_w = seed_of(config, copy, T_W)
    s_sp = seed_of(config, copy, T_SPIKE)
    # contiguous runs of rows are drawn in one call
    i = 0
    while i < len(rows):
        j = i + 1
        while j < len(rows) and rows[j] == rows[j - 1] + 1:
            j += 1
        blk = out[i:j]
        off = int(rows[i]) * K
        lib.synth_normal(s_w, off, blk.size, sigma, _fptr(blk))
        if spike_p > 0.0:
            lib.synth_spikes(s_sp, off, blk.size, spike_p, spike_mag, _fptr(blk))
        i = j
    return out


def outlier_channels(config: int, copy: int, K: int, frac: float = 0.01) -> np.ndarray:
    """round(frac*K) distinct channels: those with the smallest stream words."""
    count = int(round(frac * K))
    b = bits(seed_of(config, copy, T_OUTLIER), K)
    order = np.lexsort((np.arange(K), b))
    return np.sort(order[:count])


def activations(config: int, copy: int, M: int, K: int, *, outlier_frac: float = 0.0,
                outlier_gain: float = 20.0) -> np.ndarray:
    """fp32 x[M][K] ~ N(0,1); optional outlier channels scaled by ``outlier_gain``."""
    x = normal(seed_of(config, copy, T_X), M * K, 1.0).reshape(M, K)
    if outlier_frac > 0.0:
        ch = outlier_channels(config, copy, K, outlier_frac)
        x[:, ch] *= np.float32(outlier_gain)
    return x


# Workload recipes (shapes, distributions) of the five configurations.
PROJ_SHAPES = [(4096, 4096), (4096, 14336), (14336, 4096)]   # (K, N)

CONFIGS = {
    0: dict(name="tiny", M=[1], shapes=[(256, 128)], sigma=0.02),
    1: dict(name="decode_gemv", M=[1], shapes=PROJ_SHAPES, sigma=0.02, copies=32),
    2: dict(name="small_batch_decode", M=[4, 8, 16, 32], shapes=PROJ_SHAPES, sigma=0.02, copies=32),
    3: dict(name="prefill_gemm", M=[2048], shapes=[(4096, 14336), (14336, 4096)], sigma=0.02),
    4: dict(name="heavy_tail_stress", M=[1, 128, 4096], shapes=[(8192, 28672)], sigma=0.1,
            spike_p=0.01, spike_mag=5.0, outlier_frac=0.01, outlier_gain=20.0),
}


def config_weights(config: int, copy: int, K: int, N: int, rows=None) -> np.ndarray:
    c = CONFIGS[config]
    return weights(config, copy, N, K, rows, sigma=c["sigma"],
                   spike_p=c.get("spike_p", 0.0), spike_mag=c.get("spike_mag", 5.0))


def config_activations(config: int, copy: int, M: int, K: int) -> np.ndarray:
    c = CONFIGS[config]
    return activations(config, copy, M, K, outlier_frac=c.get("outlier_frac", 0.0),
                       outlier_gain=c.get("outlier_gain", 20.0))
