"""ORACLE -- test infrastructure only.

Python access to the plain C statement of the Sherry 3:4 ternary matmul
(``sherry_oracle.c``).  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
CUDA library never links, imports or calls it; the two share no code.

Every function cites the passage of the Sherry page (pnsm.cn/news/1195499,
"Sherry framework: ternary quantisation and 3:4 sparsity for LLM inference")
it restates:
  quantise          sec. 3.1  (min ||W - alpha T||^2 with ||T||_0 = 3 per 4)
  encode/decode     sec. 2.1  (5-bit code per group of 4, 1.25 bit/weight)
  pattern_sign      sec. 2.1 / 2.2 (4-bit pattern + 1 sign bit, 16-entry table)
  pack/unpack       sec. 2.1
  quant_act         sec. 2.2 step 1 (integer activations; the page gives no
                    rule -- per-token absmax/127, round half to even)
  gemm              sec. 1.1 / 2.2 step 4 (integer accumulation)
  gemm_lut          sec. 2.2 steps 1-4 (16-entry segment table, sign, add)
  epilogue          sec. 2.2 step 4 (float scaling after integer sums)

The second source, ``w4a8_oracle.c``, states the W4A8 FastGEMM path of the
OdysseyLLM review page (xllm-io.github.io/paper-review/blog/odysseyllm):
  w4a8_quantise     sec. 3.3  (per-channel symmetric int4, S = max|W| / 7;
                    the clipping factors gamma, beta taken as 1)
  w4a8_pack/unpack  sec. 5.2  (4-bit two's complement, two per byte)
  w4a8_sint4_to_s8  sec. 3.2 / 5.2 (shift left by 4: the int8 value 16 w)
  w4a8_gemm         sec. 3.1 / 5.2 (int8 contraction of q with 16 w in int32,
                    then divided by 16)
  w4a8_epilogue     sec. 3.1 (per-channel dequantisation after the GEMM)

Parity status of each function is listed in the header of the tests that pin
it; end to end ("is this the method") is unpinned beyond those pins because
the page prints no output values for a Sherry matmul.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsherry_oracle.so")
_lib = None

OK, BAD_ARG, BAD_SHAPE, NONFINITE, OVERFLOW = 0, 1, 2, 3, 4


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile the oracle (plain C, OpenMP over independent rows)."""
    srcs = [os.path.join(_HERE, f) for f in ("sherry_oracle.c", "w4a8_oracle.c")]
    newest = max(os.path.getmtime(f) for f in srcs)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < newest:
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
             "-fno-fast-math", "-o", _SO, *srcs, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        i64, vp = ctypes.c_int64, ctypes.c_void_p
        L.oracle_quantise.argtypes = [vp, i64, i64, vp, vp, vp]
        L.oracle_encode_group.argtypes = [vp]
        L.oracle_decode_group.argtypes = [ctypes.c_int, vp]
        L.oracle_decode_group.restype = None
        L.oracle_code_to_pattern_sign.argtypes = [ctypes.c_int, vp, vp]
        L.oracle_code_to_pattern_sign.restype = None
        L.oracle_pattern_sign_to_code.argtypes = [ctypes.c_int, ctypes.c_int]
        L.oracle_row_bytes.argtypes = [i64]
        L.oracle_row_bytes.restype = i64
        L.oracle_pack.argtypes = [vp, i64, i64, vp]
        L.oracle_unpack.argtypes = [vp, i64, i64, vp]
        L.oracle_quant_act.argtypes = [vp, i64, i64, vp, vp]
        L.oracle_gemm.argtypes = [vp, vp, i64, i64, i64, vp]
        L.oracle_gemm_lut.argtypes = [vp, vp, i64, i64, i64, vp]
        L.oracle_epilogue.argtypes = [vp, vp, vp, i64, i64, vp]
        L.oracle_epilogue.restype = None
        L.oracle_forward.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp]
        L.w4a8_oracle_quantise.argtypes = [vp, i64, i64, vp, vp]
        L.w4a8_oracle_row_bytes.argtypes = [i64]
        L.w4a8_oracle_row_bytes.restype = i64
        L.w4a8_oracle_pack.argtypes = [vp, i64, i64, vp]
        L.w4a8_oracle_unpack.argtypes = [vp, i64, i64, vp]
        L.w4a8_oracle_sint4_to_s8.argtypes = [ctypes.c_int]
        L.w4a8_oracle_gemm.argtypes = [vp, vp, i64, i64, i64, vp]
        L.w4a8_oracle_epilogue.argtypes = [vp, vp, vp, i64, i64, vp]
        L.w4a8_oracle_epilogue.restype = None
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _check(rc: int, what: str):
    if rc != OK:
        raise OracleError(f"{what}: oracle status {rc}")


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def quantise(W: np.ndarray, with_alpha64: bool = False):
    """sec. 3.1: T (int8 [N][K]) and alpha (fp32 [N]); optionally fp64 alpha."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    T = np.empty((N, K), dtype=np.int8)
    alpha = np.empty(N, dtype=np.float32)
    a64 = np.empty(N, dtype=np.float64)
    _check(_load().oracle_quantise(_p(W), N, K, _p(T), _p(alpha), _p(a64)), "quantise")
    return (T, alpha, a64) if with_alpha64 else (T, alpha)


def encode_group(t) -> int:
    t = np.ascontiguousarray(np.asarray(t, dtype=np.int8))
    return int(_load().oracle_encode_group(_p(t)))


def decode_group(code: int) -> np.ndarray:
    t = np.empty(4, dtype=np.int8)
    _load().oracle_decode_group(int(code), _p(t))
    return t


def code_to_pattern_sign(code: int):
    p, s = ctypes.c_int(), ctypes.c_int()
    _load().oracle_code_to_pattern_sign(int(code), ctypes.byref(p), ctypes.byref(s))
    return p.value, s.value


def pattern_sign_to_code(pattern4: int, sign: int) -> int:
    return int(_load().oracle_pattern_sign_to_code(int(pattern4), int(sign)))


def row_bytes(K: int) -> int:
    return int(_load().oracle_row_bytes(K))


def pack(T: np.ndarray) -> np.ndarray:
    """sec. 2.1: T [N][K] -> canonical codes [N][5K/32]."""
    T = np.ascontiguousarray(T, dtype=np.int8)
    N, K = T.shape
    codes = np.empty((N, row_bytes(K)), dtype=np.uint8)
    _check(_load().oracle_pack(_p(T), N, K, _p(codes)), "pack")
    return codes


def unpack(codes: np.ndarray, K: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N = codes.shape[0]
    T = np.empty((N, K), dtype=np.int8)
    _check(_load().oracle_unpack(_p(codes), N, K, _p(T)), "unpack")
    return T


def quant_act(x: np.ndarray):
    """Per-token absmax int8 quantisation: (q int8 [M][K], s fp32 [M])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty(M, dtype=np.float32)
    _check(_load().oracle_quant_act(_p(x), M, K, _p(q), _p(s)), "quant_act")
    return q, s


def gemm(q: np.ndarray, T: np.ndarray) -> np.ndarray:
    """acc[m][n] = sum_k q[m][k] T[n][k] (exact, int32)."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    T = np.ascontiguousarray(T, dtype=np.int8)
    M, K = q.shape
    N = T.shape[0]
    assert T.shape[1] == K
    acc = np.empty((M, N), dtype=np.int32)
    _check(_load().oracle_gemm(_p(q), _p(T), M, N, K, _p(acc)), "gemm")
    return acc


def gemm_lut(q: np.ndarray, codes: np.ndarray, K: int) -> np.ndarray:
    """sec. 2.2's table form of the same contraction, straight from codes."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    M = q.shape[0]
    N = codes.shape[0]
    acc = np.empty((M, N), dtype=np.int32)
    _check(_load().oracle_gemm_lut(_p(q), _p(codes), M, N, K, _p(acc)), "gemm_lut")
    return acc


def epilogue(acc: np.ndarray, alpha: np.ndarray, s: np.ndarray) -> np.ndarray:
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    alpha = np.ascontiguousarray(alpha, dtype=np.float32)
    s = np.ascontiguousarray(s, dtype=np.float32)
    M, N = acc.shape
    y = np.empty((M, N), dtype=np.float32)
    _load().oracle_epilogue(_p(acc), _p(alpha), _p(s), M, N, _p(y))
    return y


def forward(q: np.ndarray, s: np.ndarray, codes: np.ndarray, alpha: np.ndarray, K: int):
    """unpack -> contract -> epilogue; returns (y, acc)."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    s = np.ascontiguousarray(s, dtype=np.float32)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    alpha = np.ascontiguousarray(alpha, dtype=np.float32)
    M, N = q.shape[0], codes.shape[0]
    y = np.empty((M, N), dtype=np.float32)
    acc = np.empty((M, N), dtype=np.int32)
    _check(_load().oracle_forward(_p(q), _p(s), _p(codes), _p(alpha), M, N, K, _p(y), _p(acc)),
           "forward")
    return y, acc


def reference(x: np.ndarray, W: np.ndarray):
    """The whole path from fp32 x and W: (y, acc, q, s, codes, alpha)."""
    T, alpha = quantise(W)
    codes = pack(T)
    q, s = quant_act(x)
    y, acc = forward(q, s, codes, alpha, W.shape[1])
    return y, acc, q, s, codes, alpha


# ---- W4A8 FastGEMM (OdysseyLLM review page) ---------------------------------
W4_NOT_MULTIPLE = 5


def w4a8_quantise(W: np.ndarray):
    """sec. 3.3 with gamma = beta = 1: (W_q int8 [N][K] in [-8, 7], S fp32 [N])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    Wq = np.empty((N, K), dtype=np.int8)
    S = np.empty(N, dtype=np.float32)
    _check(_load().w4a8_oracle_quantise(_p(W), N, K, _p(Wq), _p(S)), "w4a8_quantise")
    return Wq, S


def w4a8_pack(Wq: np.ndarray) -> np.ndarray:
    """sec. 5.2: two SINT4 values per byte, even k in the low nibble."""
    Wq = np.ascontiguousarray(Wq, dtype=np.int8)
    N, K = Wq.shape
    out = np.empty((N, int(_load().w4a8_oracle_row_bytes(K))), dtype=np.uint8)
    _check(_load().w4a8_oracle_pack(_p(Wq), N, K, _p(out)), "w4a8_pack")
    return out


def w4a8_unpack(packed: np.ndarray, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    Wq = np.empty((N, K), dtype=np.int8)
    _check(_load().w4a8_oracle_unpack(_p(packed), N, K, _p(Wq)), "w4a8_unpack")
    return Wq


def w4a8_sint4_to_s8(nibble: int) -> int:
    """sec. 3.2 / 5.2: the 4 bits shifted into the high half of an int8."""
    return int(_load().w4a8_oracle_sint4_to_s8(int(nibble)))


def w4a8_gemm(q: np.ndarray, packed: np.ndarray, K: int) -> np.ndarray:
    """sec. 3.1 / 5.2: acc = (sum_k q[m][k] * SINT4toS8(w[n][k])) / 16, int32."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    M, N = q.shape[0], packed.shape[0]
    acc = np.empty((M, N), dtype=np.int32)
    _check(_load().w4a8_oracle_gemm(_p(q), _p(packed), M, N, K, _p(acc)), "w4a8_gemm")
    return acc


def w4a8_epilogue(acc: np.ndarray, S: np.ndarray, s: np.ndarray) -> np.ndarray:
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    S = np.ascontiguousarray(S, dtype=np.float32)
    s = np.ascontiguousarray(s, dtype=np.float32)
    M, N = acc.shape
    y = np.empty((M, N), dtype=np.float32)
    _load().w4a8_oracle_epilogue(_p(acc), _p(S), _p(s), M, N, _p(y))
    return y


def w4a8_forward(q: np.ndarray, s: np.ndarray, packed: np.ndarray, S: np.ndarray, K: int):
    """contract -> divide by 16 -> dequantise; returns (y, acc)."""
    acc = w4a8_gemm(q, packed, K)
    return w4a8_epilogue(acc, S, s), acc


def w4a8_reference(x: np.ndarray, W: np.ndarray):
    """The whole W4A8 path from fp32 x and W: (y, acc, q, s, packed, S)."""
    Wq, S = w4a8_quantise(W)
    packed = w4a8_pack(Wq)
    q, s = quant_act(x)
    y, acc = w4a8_forward(q, s, packed, S, W.shape[1])
    return y, acc, q, s, packed, S
