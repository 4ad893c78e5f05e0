"""Host half of the W4A8 FastGEMM entry points (no GPU): sizes, the host
packer and unpacker against the oracle byte for byte (OdysseyLLM review page,
xllm-io.github.io/paper-review/blog/odysseyllm, sec. 3.3 and 5.2), and the
argument errors every call returns before it launches anything."""
import ctypes

import numpy as np
import pytest

import oracle
import sparse_bit_matmul_b200 as sbm
import synth


def test_w4a8_sizes(lib):
    assert sbm.w4a8_packed_bytes(4096, 14336) == 4096 * 14336 // 2
    assert sbm.w4a8_native_bytes(128, 128) == 8192
    assert sbm.w4a8_native_bytes(129, 160) == 2 * 2 * 8192
    assert sbm.w4a8_native_bytes(14336, 4096) == 112 * 32 * 8192
    assert sbm.w4a8_packed_bytes(10, 100) == 0                    # K % 32 != 0
    assert sbm.w4a8_packed_bytes(1, 132096) == 66048              # the largest K (a multiple of 32)
    assert sbm.w4a8_native_bytes(1, 132128) == 0                  # past it


@pytest.mark.parametrize("N,K,cfg", [(128, 256, 0), (37, 96, 0), (300, 4096, 1), (64, 8192, 4)])
def test_w4a8_pack_equals_oracle(N, K, cfg, lib):
    W = synth.config_weights(cfg, 0, K, N)
    w4, scale = sbm.w4a8_pack(W)
    Wq, S = oracle.w4a8_quantise(W)
    assert np.array_equal(scale.view(np.uint32), S.view(np.uint32))
    assert np.array_equal(w4, oracle.w4a8_pack(Wq))
    assert np.array_equal(sbm.w4a8_unpack(w4, K), Wq)


def test_w4a8_pack_edge_rows(lib):
    W = np.zeros((5, 32), dtype=np.float32)
    W[1] = -0.25                                   # all negative, equal
    W[2, :8] = [7.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 6.5]   # S = 1: exact ties
    W[3] = np.float32(1e-38)                       # tiny values
    W[4, 0] = -3.0                                 # one nonzero
    w4, scale = sbm.w4a8_pack(W)
    Wq, S = oracle.w4a8_quantise(W)
    assert np.array_equal(w4, oracle.w4a8_pack(Wq)) and np.array_equal(scale, S)
    assert scale[0] == 0 and not w4[0].any()


def test_w4a8_unpack_any_bytes(lib):
    raw = np.random.default_rng(3).integers(0, 256, size=(9, 64), dtype=np.uint8)
    assert np.array_equal(sbm.w4a8_unpack(raw, 128), oracle.w4a8_unpack(raw, 128))


def test_w4a8_argument_errors(lib):
    L = lib.load()
    W = np.ones((4, 32), dtype=np.float32)
    w4 = np.empty((4, 16), dtype=np.uint8)
    S = np.empty(4, dtype=np.float32)
    assert L.sherry_w4a8_pack(None, 4, 32, w4.ctypes.data, S.ctypes.data) == sbm.ERR_INVALID_ARG
    assert L.sherry_w4a8_pack(W.ctypes.data, 4, 20, w4.ctypes.data, S.ctypes.data) == sbm.ERR_UNSUPPORTED_SHAPE
    W[2, 3] = np.inf
    assert L.sherry_w4a8_pack(W.ctypes.data, 4, 32, w4.ctypes.data, S.ctypes.data) == sbm.ERR_NONFINITE
    with pytest.raises(sbm.SherryError):
        sbm.w4a8_pack(np.full((2, 32), np.nan, dtype=np.float32))
    assert L.sherry_w4a8_repack(None, 1, 32, None, None) == sbm.ERR_INVALID_ARG
    fake = ctypes.c_void_p(1 << 20)
    assert L.sherry_w4a8_repack(fake, 1, 132128, fake, None) == sbm.ERR_UNSUPPORTED_SHAPE
    assert L.sherry_w4a8_gemm(None, None, None, None, None, 1, 1, 32, None) == sbm.ERR_INVALID_ARG
    assert L.sherry_w4a8_gemm(fake, fake, fake, fake, fake, 1, 1, 33, None) == sbm.ERR_UNSUPPORTED_SHAPE
    assert L.sherry_w4a8_gemm(fake, fake, fake, fake, fake, 1, 1, 132128, None) == sbm.ERR_UNSUPPORTED_SHAPE
    assert L.sherry_w4a8_gemm_acc(fake, fake, fake, fake, None, None, 1, 1, 32, None) == sbm.ERR_INVALID_ARG
    assert L.sherry_w4a8_gemm(ctypes.c_void_p((1 << 20) + 4), fake, fake, fake, fake, 1, 1, 32, None) == \
        sbm.ERR_INVALID_ARG
    # the GEMV serves M <= 4 only; both explicit kernels check shapes before launching
    assert L.sherry_w4a8_gemm_gemv(fake, fake, fake, fake, fake, None, sbm.W4A8_GEMV_MAX_M + 1, 1, 32, None) == \
        sbm.ERR_UNSUPPORTED_SHAPE
    assert L.sherry_w4a8_gemm_gemv(fake, fake, fake, fake, fake, None, 1, 1, 132128, None) == \
        sbm.ERR_UNSUPPORTED_SHAPE
    assert L.sherry_w4a8_gemm_tc(fake, fake, fake, fake, fake, None, 1, 1, 48, None) == sbm.ERR_UNSUPPORTED_SHAPE
    assert L.sherry_w4a8_gemm_tc(None, fake, fake, fake, fake, None, 1, 1, 32, None) == sbm.ERR_INVALID_ARG


def test_w4a8_linear_wiring(lib, monkeypatch):
    """W4A8Linear marshals the host pack, the device repack, the quantiser
    and the GEMM in that order (device calls replaced by recorders)."""
    import torch
    calls = []
    monkeypatch.setattr(sbm, "w4a8_repack", lambda w4_dev, N, K: calls.append(("repack", tuple(w4_dev.shape), N, K))
                        or "native")
    monkeypatch.setattr(sbm, "quant_act", lambda x: calls.append(("quant", tuple(x.shape))) or ("q", "s"))
    monkeypatch.setattr(sbm, "w4a8_gemm", lambda q, s, nat, sc, N, out=None:
                        calls.append(("gemm", q, s, nat, tuple(sc.shape), N, out)) or "y")
    W = synth.weights(0, 7, 40, 96)
    layer = sbm.W4A8Linear.from_weights(W, device="cpu")
    w4, S = oracle.w4a8_pack(oracle.w4a8_quantise(W)[0]), oracle.w4a8_quantise(W)[1]
    assert np.array_equal(layer.scale.numpy(), S) and (layer.N, layer.K) == (40, 96)
    assert layer.forward(torch.zeros(3, 96)) == "y"
    assert calls == [("repack", w4.shape, 40, 96), ("quant", (3, 96)), ("gemm", "q", "s", "native", (40,), 40, None)]
