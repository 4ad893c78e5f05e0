"""Python binding of libsherry_b200 (include/sherry.h): the Sherry 3:4 ternary
matmul on B200.

Only argument marshalling lives here: every step of the path runs in the C /
CUDA library.  Host functions take numpy arrays; device functions take torch
CUDA tensors (torch supplies device memory and the current stream).  There
is no fallback: if the library is missing or a call fails, an exception is
raised.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SO_PATH = os.path.join(HERE, "libsherry_b200.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_NONFINITE, ERR_CUDA, ERR_DEVICE, ERR_WORKSPACE = range(7)

# every entry point declared in include/sherry.h
ABI_SYMBOLS = (
    "sherry_status_string", "sherry_version", "sherry_packed_bytes", "sherry_native_bytes",
    "sherry_pack", "sherry_unpack", "sherry_repack", "sherry_quant_act", "sherry_gemm",
    "sherry_gemm_acc", "sherry_gemm_tc", "sherry_gemm_gemv", "sherry_gemm_simt", "sherry_gemm_noalloc",
    "sherry_gemm_decode", "sherry_linear", "sherry_linear_ex", "sherry_last_device_status",
    "sherry_workspace_bytes", "sherry_reserve", "sherry_selftest_wait",
    "sherry_w4a8_packed_bytes", "sherry_w4a8_native_bytes", "sherry_w4a8_pack", "sherry_w4a8_unpack",
    "sherry_w4a8_repack", "sherry_w4a8_gemm", "sherry_w4a8_gemm_acc", "sherry_w4a8_gemm_tc",
    "sherry_w4a8_gemm_gemv",
)

_lib = None


class SherryError(RuntimeError):
    def __init__(self, what: str, status: int):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def load() -> ctypes.CDLL:
    """Load the in-tree library; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(SO_PATH):
        raise ImportError(f"{SO_PATH} is missing: run `python -m sparse_bit_matmul_b200.build`")
    L = ctypes.CDLL(SO_PATH)
    i64, vp, c_int = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
    L.sherry_status_string.argtypes = [c_int]
    L.sherry_status_string.restype = ctypes.c_char_p
    L.sherry_version.restype = c_int
    L.sherry_packed_bytes.argtypes = [i64, i64]
    L.sherry_packed_bytes.restype = ctypes.c_size_t
    L.sherry_native_bytes.argtypes = [i64, i64]
    L.sherry_native_bytes.restype = ctypes.c_size_t
    L.sherry_pack.argtypes = [vp, i64, i64, vp, vp]
    L.sherry_unpack.argtypes = [vp, i64, i64, vp]
    L.sherry_repack.argtypes = [vp, i64, i64, vp, vp]
    L.sherry_quant_act.argtypes = [vp, i64, i64, vp, vp, vp]
    L.sherry_gemm.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.sherry_gemm_acc.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.sherry_gemm_simt.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.sherry_gemm_tc.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.sherry_gemm_gemv.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.sherry_gemm_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.sherry_gemm_decode.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.sherry_linear.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp]
    L.sherry_linear_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.sherry_last_device_status.argtypes = [c_int]
    L.sherry_workspace_bytes.argtypes = [i64, i64]
    L.sherry_workspace_bytes.restype = ctypes.c_size_t
    L.sherry_reserve.argtypes = [i64, i64]
    L.sherry_selftest_wait.argtypes = [ctypes.c_uint64, vp]
    L.sherry_w4a8_packed_bytes.argtypes = [i64, i64]
    L.sherry_w4a8_packed_bytes.restype = ctypes.c_size_t
    L.sherry_w4a8_native_bytes.argtypes = [i64, i64]
    L.sherry_w4a8_native_bytes.restype = ctypes.c_size_t
    L.sherry_w4a8_pack.argtypes = [vp, i64, i64, vp, vp]
    L.sherry_w4a8_unpack.argtypes = [vp, i64, i64, vp]
    L.sherry_w4a8_repack.argtypes = [vp, i64, i64, vp, vp]
    L.sherry_w4a8_gemm.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.sherry_w4a8_gemm_acc.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.sherry_w4a8_gemm_tc.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.sherry_w4a8_gemm_gemv.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp]
    for name in ABI_SYMBOLS:
        getattr(L, name).restype = getattr(L, name).restype or c_int
    _lib = L
    return L


def status_string(status: int) -> str:
    return load().sherry_status_string(int(status)).decode()


def _check(rc: int, what: str):
    if rc != OK:
        raise SherryError(what, rc)


def _np_ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _dptr(t):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "device arguments must be contiguous CUDA tensors"
    return t.data_ptr()


def _stream(t):
    import torch
    return torch.cuda.current_stream(t.device).cuda_stream


# ----------------------------------------------------------------- host side
def packed_bytes(N: int, K: int) -> int:
    return int(load().sherry_packed_bytes(N, K))


def native_bytes(N: int, K: int) -> int:
    return int(load().sherry_native_bytes(N, K))


def pack(W: np.ndarray):
    """fp32 W [N][K] -> (canonical codes uint8 [N][5K/32], alpha fp32 [N])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    codes = np.empty((N, K // 32 * 5), dtype=np.uint8)
    alpha = np.empty(N, dtype=np.float32)
    _check(load().sherry_pack(_np_ptr(W), N, K, _np_ptr(codes), _np_ptr(alpha)), "sherry_pack")
    return codes, alpha


def unpack(codes: np.ndarray, K: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N = codes.shape[0]
    T = np.empty((N, K), dtype=np.int8)
    _check(load().sherry_unpack(_np_ptr(codes), N, K, _np_ptr(T)), "sherry_unpack")
    return T


# --------------------------------------------------------------- device side
_reserved = {}          # device index -> (max_M, max_K) reserved through this binding


def workspace_bytes(max_M: int, max_K: int) -> int:
    """Device bytes sherry_reserve(max_M, max_K) sets aside on the current device."""
    return int(load().sherry_workspace_bytes(max_M, max_K))


def reserve(max_M: int, max_K: int, device=None):
    """sherry_reserve on `device` (default: the current CUDA device): host-
    synchronous; sets aside the workspace of every later call with
    M <= max_M and K <= max_K.  Call it before capturing CUDA graphs."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    idx = dev.index if dev.index is not None else torch.cuda.current_device()
    m0, k0 = _reserved.get(idx, (0, 0))
    m1, k1 = max(m0, int(max_M)), max(k0, int(max_K))
    if (m1, k1) != (m0, k0):
        with torch.cuda.device(idx):
            _check(load().sherry_reserve(m1, k1), "sherry_reserve")
        _reserved[idx] = (m1, k1)


def _ensure_workspace(t, M: int, K: int):
    # the asynchronous entry points never allocate: the binding reserves (host,
    # synchronous) the first time a call needs more than was set aside
    m0, k0 = _reserved.get(t.device.index, (0, 0))
    if M > m0 or K > k0:
        reserve(M, K, t.device)


def repack(codes_dev, N: int, K: int, out=None):
    """Canonical codes on the device -> kernel-native layout (uint8 tensor)."""
    import torch
    if out is None:
        out = torch.empty(native_bytes(N, K), dtype=torch.uint8, device=codes_dev.device)
    _check(load().sherry_repack(_dptr(codes_dev), N, K, _dptr(out), _stream(codes_dev)), "sherry_repack")
    return out


def quant_act(x, out_q=None, out_s=None):
    """fp32 x [M][K] -> (int8 [M][K], fp32 scale [M])."""
    import torch
    M, K = x.shape
    q = out_q if out_q is not None else torch.empty((M, K), dtype=torch.int8, device=x.device)
    s = out_s if out_s is not None else torch.empty(M, dtype=torch.float32, device=x.device)
    _check(load().sherry_quant_act(_dptr(x), M, K, _dptr(q), _dptr(s), _stream(x)), "sherry_quant_act")
    return q, s


GEMV_MAX_M = 4      # SHERRY_GEMV_MAX_M
DECODE_MAX_M = 8    # SHERRY_DECODE_MAX_M
GEMM_DECODE_AUTO_MAX_M = 2   # SHERRY_GEMM_DECODE_AUTO_MAX_M
LINEAR_FUSED_MAX_M = 1   # SHERRY_LINEAR_FUSED_MAX_M


def gemm(x_i8, x_scale, w_native, alpha, N: int, out=None, acc=None, want_y: bool = True,
         kernel: str = "auto"):
    """y fp32 [M][N] (and optionally exact int32 acc) from int8 activations and
    kernel-native codes.  kernel: "auto" (sherry_gemm: the decode kernel
    for M <= 2, tensor cores above), "decode", "tc", "gemv" (the page's
    table lookup), "simt" (comparison kernel) or "noalloc"."""
    import torch
    M, K = x_i8.shape
    y = None
    if want_y:
        y = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=x_i8.device)
    L = load()
    if kernel != "noalloc":
        _ensure_workspace(x_i8, M, K)
    args = (_dptr(x_i8), _dptr(x_scale), _dptr(w_native), _dptr(alpha), _dptr(y), _dptr(acc), M, N, K,
            _stream(x_i8))
    if kernel == "auto":
        if acc is None:
            rc = L.sherry_gemm(args[0], args[1], args[2], args[3], args[4], M, N, K, args[-1])
        else:
            rc = L.sherry_gemm_acc(*args)
    elif kernel == "tc":
        rc = L.sherry_gemm_tc(*args)
    elif kernel == "gemv":
        rc = L.sherry_gemm_gemv(*args)
    elif kernel == "simt":
        rc = L.sherry_gemm_simt(*args)
    elif kernel == "noalloc":
        rc = L.sherry_gemm_noalloc(*args)
    elif kernel == "decode":
        rc = L.sherry_gemm_decode(*args)
    else:
        raise ValueError(kernel)
    _check(rc, f"sherry_gemm[{kernel}]")
    return y


def linear(x, w_native, alpha, N: int, out=None, acc=None, out_q=None, out_s=None, want_y: bool = True):
    """y fp32 [M][N] straight from fp32 activations x [M][K] (sherry_linear:
    quantiser + GEMM, one launch for M = 1).  Optional acc int32 [M][N] and
    out_q int8 [M][K] / out_s fp32 [M] receive the exact accumulators and the
    quantised activations."""
    import torch
    M, K = x.shape
    y = None
    if want_y:
        y = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=x.device)
    L = load()
    _ensure_workspace(x, M, K)
    if acc is None and out_q is None and out_s is None:
        rc = L.sherry_linear(_dptr(x), _dptr(w_native), _dptr(alpha), _dptr(y), M, N, K, _stream(x))
    else:
        rc = L.sherry_linear_ex(_dptr(x), _dptr(w_native), _dptr(alpha), _dptr(y), _dptr(acc), _dptr(out_q),
                                _dptr(out_s), M, N, K, _stream(x))
    _check(rc, "sherry_linear")
    return y


def last_device_status(reset: bool = False) -> int:
    return int(load().sherry_last_device_status(1 if reset else 0))


DEV_TIMEOUT_SELFTEST = 0x107   # device status code of sherry_selftest_wait


def selftest_wait(limit_ns: int, stream=None):
    """sherry_selftest_wait on the current stream: a bounded wait that runs out."""
    import torch
    st = torch.cuda.current_stream().cuda_stream if stream is None else stream
    _check(load().sherry_selftest_wait(int(limit_ns), st), "sherry_selftest_wait")


class PackedLinear:
    """Weights of one Sherry linear layer resident on the device.

    ``PackedLinear.from_weights(W)`` packs on the host (sherry_pack), copies
    the canonical codes and alpha to the device and repacks them into the
    kernel-native layout.  ``forward(x)`` quantises the activations and runs
    the GEMM (sherry_linear), asynchronously on the current stream.
    """

    def __init__(self, w_native, alpha, N: int, K: int):
        self.w_native, self.alpha, self.N, self.K = w_native, alpha, N, K

    @classmethod
    def from_weights(cls, W: np.ndarray, device="cuda"):
        import torch
        codes, alpha = pack(W)
        return cls.from_codes(codes, alpha, W.shape[1], device)

    @classmethod
    def from_codes(cls, codes: np.ndarray, alpha: np.ndarray, K: int, device="cuda"):
        import torch
        N = codes.shape[0]
        codes_d = torch.from_numpy(codes).to(device)
        w_native = repack(codes_d, N, K)
        return cls(w_native, torch.from_numpy(alpha).to(device), N, K)

    def forward(self, x, out=None):
        return linear(x, self.w_native, self.alpha, self.N, out=out)


# ------------------------------------------------ W4A8 FastGEMM (SINT4 x int8)
def w4a8_packed_bytes(N: int, K: int) -> int:
    return int(load().sherry_w4a8_packed_bytes(N, K))


def w4a8_native_bytes(N: int, K: int) -> int:
    return int(load().sherry_w4a8_native_bytes(N, K))


def w4a8_pack(W: np.ndarray):
    """fp32 W [N][K] -> (canonical SINT4 rows uint8 [N][K/2], per-channel scale fp32 [N])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    w4 = np.empty((N, K // 2), dtype=np.uint8)
    scale = np.empty(N, dtype=np.float32)
    _check(load().sherry_w4a8_pack(_np_ptr(W), N, K, _np_ptr(w4), _np_ptr(scale)), "sherry_w4a8_pack")
    return w4, scale


def w4a8_unpack(w4: np.ndarray, K: int) -> np.ndarray:
    w4 = np.ascontiguousarray(w4, dtype=np.uint8)
    N = w4.shape[0]
    Wq = np.empty((N, K), dtype=np.int8)
    _check(load().sherry_w4a8_unpack(_np_ptr(w4), N, K, _np_ptr(Wq)), "sherry_w4a8_unpack")
    return Wq


def w4a8_repack(w4_dev, N: int, K: int, out=None):
    """Canonical SINT4 rows on the device -> kernel-native layout (uint8 tensor)."""
    import torch
    if out is None:
        out = torch.empty(w4a8_native_bytes(N, K), dtype=torch.uint8, device=w4_dev.device)
    _check(load().sherry_w4a8_repack(_dptr(w4_dev), N, K, _dptr(out), _stream(w4_dev)), "sherry_w4a8_repack")
    return out


W4A8_GEMV_MAX_M = 4   # SHERRY_W4A8_GEMV_MAX_M


def w4a8_gemm(x_i8, x_scale, w4_native, scale, N: int, out=None, acc=None, want_y: bool = True,
              kernel: str = "auto"):
    """y fp32 [M][N] (and optionally the int32 sums after the division by 16)
    from int8 activations and kernel-native SINT4 weights.  kernel: "auto"
    (sherry_w4a8_gemm: the tensor-core kernel for every M), "tc" or "gemv"
    (the CUDA-core comparison kernel, M <= 4)."""
    import torch
    M, K = x_i8.shape
    y = None
    if want_y:
        y = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=x_i8.device)
    L = load()
    _ensure_workspace(x_i8, M, K)
    args = (_dptr(x_i8), _dptr(x_scale), _dptr(w4_native), _dptr(scale), _dptr(y), _dptr(acc), M, N, K,
            _stream(x_i8))
    if kernel == "auto":
        if acc is None:
            rc = L.sherry_w4a8_gemm(args[0], args[1], args[2], args[3], args[4], M, N, K, args[-1])
        else:
            rc = L.sherry_w4a8_gemm_acc(*args)
    elif kernel == "tc":
        rc = L.sherry_w4a8_gemm_tc(*args)
    elif kernel == "gemv":
        rc = L.sherry_w4a8_gemm_gemv(*args)
    else:
        raise ValueError(kernel)
    _check(rc, f"sherry_w4a8_gemm[{kernel}]")
    return y


class W4A8Linear:
    """Weights of one W4A8 linear layer resident on the device.

    ``W4A8Linear.from_weights(W)`` quantises and packs on the host
    (sherry_w4a8_pack), copies the SINT4 rows and the channel scales to the
    device and repacks them (sherry_w4a8_repack).  ``forward(x)`` quantises
    the activations (sherry_quant_act) and runs the W4A8 GEMM
    (sherry_w4a8_gemm), asynchronously on the current stream.
    """

    def __init__(self, w_native, scale, N: int, K: int):
        self.w_native, self.scale, self.N, self.K = w_native, scale, N, K

    @classmethod
    def from_weights(cls, W: np.ndarray, device="cuda"):
        import torch
        w4, scale = w4a8_pack(W)
        N, K = W.shape
        w_native = w4a8_repack(torch.from_numpy(w4).to(device), N, K)
        return cls(w_native, torch.from_numpy(scale).to(device), N, K)

    def forward(self, x, out=None):
        q, s = quant_act(x)
        return w4a8_gemm(q, s, self.w_native, self.scale, self.N, out=out)
