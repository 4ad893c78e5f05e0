"""The CPU comparison kernel (the Sherry page's x86 table-lookup scheme,
sec. 2.2 steps 1-4 and sec. 5.1) against the oracle: int32 sums and fp32
outputs bit for bit, on the AVX2 path and on the plain-C path."""
import numpy as np
import pytest

import cpu_lut
import oracle
import synth

SHAPES = [(1, 128, 256), (3, 37, 96), (2, 100, 4096), (1, 65, 14336), (4, 33, 2048), (1, 4096, 4096)]


@pytest.mark.parametrize("path", ["avx2", "scalar"])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_lut_equals_oracle(M, N, K, path):
    if path == "avx2" and not cpu_lut.has_avx2():
        pytest.skip("no AVX2 on this host")
    W = synth.weights(0, 5, N, K, sigma=0.02)
    x = synth.activations(0, 5, M, K)
    y_o, acc_o, q_o, s_o, codes_o, alpha_o = oracle.reference(x, W)
    prep = cpu_lut.prepare(codes_o, K)
    y, acc = cpu_lut.gemm(q_o, s_o, prep, alpha_o, N, K, force_scalar=(path == "scalar"))
    assert np.array_equal(acc, acc_o)
    assert np.array_equal(y.view(np.uint32), y_o.view(np.uint32))


def test_lut_extreme_activations_every_code():
    """All 32 codes in every row position, activations at +-127: the largest
    table entries (+-381) and int16 runs of 64 groups near their limit."""
    K, N = 32 * 64, 40
    codes_T = np.array([oracle.decode_group(c) for c in range(32)], dtype=np.int8)     # [32][4]
    rng = np.random.default_rng(2)
    T = codes_T[rng.integers(0, 32, size=(N, K // 4))].reshape(N, K)
    T[0] = np.tile(codes_T[31], K // 4)                       # one row of the same code
    codes = oracle.pack(T)
    q = np.where(rng.random((2, K)) < 0.5, -127, 127).astype(np.int8)
    q[0] = 127
    s = np.array([0.5, 0.25], dtype=np.float32)
    alpha = np.full(N, 0.125, dtype=np.float32)
    acc_o = oracle.gemm(q, T)
    y_o = oracle.epilogue(acc_o, alpha, s)
    prep = cpu_lut.prepare(codes, K)
    for scalar in (False, True):
        if not scalar and not cpu_lut.has_avx2():
            continue
        y, acc = cpu_lut.gemm(q, s, prep, alpha, N, K, force_scalar=scalar)
        assert np.array_equal(acc, acc_o) and np.array_equal(y, y_o)
