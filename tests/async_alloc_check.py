"""Run by tests/test_gpu_boundary.py in a child process with
CUDA_MODULE_LOADING=EAGER, so that every kernel of the library is loaded when
the context is created: the device's free memory then moves only if the
library itself allocates.  Device buffers come from cuda-python (no torch in
this process).  After sherry_reserve(64, 8192), first calls on fresh shapes
of every asynchronous entry point family (decode kernel, fused linear,
tensor cores with split tiles, two-launch linear, W4A8) must leave
cudaMemGetInfo unchanged, and the int32 accumulators must equal the
oracle's.  Prints "ok" and exits 0, or prints what failed and exits 1."""
import ctypes
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from cuda.bindings import runtime as cudart  # noqa: E402

import oracle  # noqa: E402
import synth  # noqa: E402


def ck(ret):
    err = ret[0] if isinstance(ret, tuple) else ret
    if err != cudart.cudaError_t.cudaSuccess:
        raise RuntimeError(f"CUDA error {err}")
    return ret[1] if isinstance(ret, tuple) and len(ret) == 2 else ret


def dev_alloc(nbytes):
    return ck(cudart.cudaMalloc(max(int(nbytes), 16)))


def to_dev(a: np.ndarray):
    a = np.ascontiguousarray(a)
    p = dev_alloc(a.nbytes)
    ck(cudart.cudaMemcpy(p, a.ctypes.data, a.nbytes, cudart.cudaMemcpyKind.cudaMemcpyHostToDevice))
    return p


def from_dev(p, shape, dtype):
    out = np.empty(shape, dtype=dtype)
    ck(cudart.cudaMemcpy(out.ctypes.data, p, out.nbytes, cudart.cudaMemcpyKind.cudaMemcpyDeviceToHost))
    return out


def main():
    ck(cudart.cudaSetDevice(0))
    L = ctypes.CDLL(os.path.join(ROOT, "sparse_bit_matmul_b200", "libsherry_b200.so"))
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    for name in ("sherry_gemm_acc", "sherry_gemm_tc"):
        getattr(L, name).argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.sherry_quant_act.argtypes = [vp, i64, i64, vp, vp, vp]
    L.sherry_linear.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp]
    L.sherry_w4a8_gemm.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp]
    L.sherry_pack.argtypes = [vp, i64, i64, vp, vp]
    L.sherry_w4a8_pack.argtypes = [vp, i64, i64, vp, vp]
    L.sherry_repack.argtypes = [vp, i64, i64, vp, vp]
    L.sherry_w4a8_repack.argtypes = [vp, i64, i64, vp, vp]
    L.sherry_native_bytes.argtypes = [i64, i64]
    L.sherry_native_bytes.restype = ctypes.c_size_t
    L.sherry_w4a8_native_bytes.argtypes = [i64, i64]
    L.sherry_w4a8_native_bytes.restype = ctypes.c_size_t
    L.sherry_reserve.argtypes = [i64, i64]
    if L.sherry_reserve(64, 8192) != 0:
        print("sherry_reserve failed")
        return 1
    cases = [(1, 4096, 4096), (3, 300, 4096), (16, 256, 8192), (40, 1000, 1024), (64, 640, 2048)]
    prepared = []
    for M, N, K in cases:
        W = synth.weights(8, M, N, K)
        x = synth.activations(8, M, M, K)
        codes = np.empty((N, K // 32 * 5), dtype=np.uint8)
        alpha = np.empty(N, dtype=np.float32)
        assert L.sherry_pack(W.ctypes.data, N, K, codes.ctypes.data, alpha.ctypes.data) == 0
        w4 = np.empty((N, K // 2), dtype=np.uint8)
        S4 = np.empty(N, dtype=np.float32)
        assert L.sherry_w4a8_pack(W.ctypes.data, N, K, w4.ctypes.data, S4.ctypes.data) == 0
        codes_d, w4_d = to_dev(codes), to_dev(w4)
        nat = dev_alloc(L.sherry_native_bytes(N, K))
        nat4 = dev_alloc(L.sherry_w4a8_native_bytes(N, K))
        assert L.sherry_repack(codes_d, N, K, nat, None) == 0
        assert L.sherry_w4a8_repack(w4_d, N, K, nat4, None) == 0
        bufs = dict(x=to_dev(x), alpha=to_dev(alpha), S4=to_dev(S4), q=dev_alloc(M * K), s=dev_alloc(4 * M),
                    y=dev_alloc(4 * M * N), y2=dev_alloc(4 * M * N), acc=dev_alloc(4 * M * N),
                    acc2=dev_alloc(4 * M * N))
        prepared.append((M, N, K, W, x, nat, nat4, bufs))
    ck(cudart.cudaDeviceSynchronize())
    err, free0, _ = cudart.cudaMemGetInfo()
    ck(err)
    for M, N, K, W, x, nat, nat4, b in prepared:
        assert L.sherry_quant_act(b["x"], M, K, b["q"], b["s"], None) == 0
        assert L.sherry_gemm_acc(b["q"], b["s"], nat, b["alpha"], b["y"], b["acc"], M, N, K, None) == 0
        assert L.sherry_gemm_tc(b["q"], b["s"], nat, b["alpha"], b["y"], b["acc2"], M, N, K, None) == 0
        assert L.sherry_linear(b["x"], nat, b["alpha"], b["y2"], M, N, K, None) == 0
        assert L.sherry_w4a8_gemm(b["q"], b["s"], nat4, b["S4"], b["y"], M, N, K, None) == 0
    ck(cudart.cudaDeviceSynchronize())
    err, free1, _ = cudart.cudaMemGetInfo()
    ck(err)
    if free1 != free0:
        print(f"free device memory changed: {free0} -> {free1}")
        return 1
    for M, N, K, W, x, nat, nat4, b in prepared:
        _, acc_o, *_ = oracle.reference(x, W)
        for key in ("acc", "acc2"):
            if not np.array_equal(from_dev(b[key], (M, N), np.int32), acc_o):
                print(f"{key} differs from the oracle at M={M} N={N} K={K}")
                return 1
    print("ok")
    return 0


if __name__ == "__main__":
    sys.exit(main())
