"""Pins of the oracle against what the Sherry page and mathematics fix.

Each test ties one oracle function to something other than itself:
  quantise        brute force over all 32 (K=4) and 32^2 (K=8, shared alpha)
                  3:4 ternary patterns; the closed-form error identity; tie and
                  signed-zero rules; the page's example block (golden file)
  encode/decode   exhaustive over the 32 codes; exactly 3 nonzeros each (the
                  page's "keep the 3:4 sparsity strictly" check)
  pattern/sign    the page's 16-entry pattern + sign bit form is a bijection
                  and negating the sign bit negates the group
  pack/unpack     bits read back one by one at all 8 bit offsets; random
                  streams round trip both ways (every 5-bit value is a code)
  gemm            numpy int64 matmul (a library routine) and the page's
                  16-entry table form of the contraction
  quant_act       range, argmax -> +-127, half-step error bound, half-to-even
                  ties on exactly constructed inputs, the all-zero token
  epilogue        fp64 bound of two rounded products; exact when the scales
                  are powers of two
Sources: Sherry page (pnsm.cn/news/1195499) sec. 1.1, 2.1, 2.2, 3.1, 6.1.
"""
import itertools
import json
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def all_34_patterns():
    """All vectors in {-1,0,1}^4 with exactly three nonzeros (brute force)."""
    pats = [np.array(v, dtype=np.int64) for v in itertools.product((-1, 0, 1), repeat=4)
            if sum(1 for e in v if e != 0) == 3]
    assert len(pats) == 32
    return np.stack(pats)


def err_of(W, T, alpha):
    W = W.astype(np.float64)
    return float(((W - alpha * T.astype(np.float64)) ** 2).sum())


# ---------------------------------------------------------------- quantise
def test_quantise_bruteforce_K4():
    rng = np.random.default_rng(1234)
    P = all_34_patterns().astype(np.float64)          # [32][4]
    rows = rng.normal(0, 1, size=(10000, 4)).astype(np.float32)
    # hand-built ties, zeros and signed zeros
    extra = np.array([[0.5, 0.5, 0.5, 0.5], [0, 0, 0, 0], [-0.0, 1, -1, 2],
                      [1, -1, 1, -1], [3, 0, 0, 3], [-2, -2, 1, 1],
                      [0.25, -0.25, 0.25, 0.0]], dtype=np.float32)
    rows = np.concatenate([rows, extra])
    # each 4-element row is its own N=1, K=4 problem (alpha per row)
    Tq, al, al64 = oracle.quantise(rows, with_alpha64=True)
    Wd = rows.astype(np.float64)
    ip = Wd @ P.T                                       # [R][32]
    best = (Wd ** 2).sum(1) - np.maximum(ip, 0).max(1) ** 2 / 3.0
    got = np.array([err_of(rows[i], Tq[i], al64[i]) for i in range(len(rows))])
    scale = np.maximum((Wd ** 2).sum(1), 1e-300)
    assert np.all(np.abs(got - best) <= 1e-12 * scale + 1e-300)
    # alpha is the least-squares scale for the chosen T
    assert np.allclose(al64, (Wd * Tq).sum(1) / 3.0, rtol=0, atol=1e-15)


def test_quantise_bruteforce_K8_shared_alpha():
    rng = np.random.default_rng(99)
    P = all_34_patterns().astype(np.float64)
    P8 = np.concatenate([np.repeat(P, 32, 0), np.tile(P, (32, 1))], 1)   # [1024][8]
    rows = rng.standard_t(3, size=(2000, 8)).astype(np.float32)
    Tq, al, al64 = oracle.quantise(rows, with_alpha64=True)
    Wd = rows.astype(np.float64)
    best = (Wd ** 2).sum(1) - np.maximum(Wd @ P8.T, 0).max(1) ** 2 / 6.0
    got = np.array([err_of(rows[i], Tq[i], al64[i]) for i in range(len(rows))])
    assert np.all(np.abs(got - best) <= 1e-12 * (Wd ** 2).sum(1))


def test_quantise_closed_form_identity_full_rows():
    W = synth.weights(1, 0, 64, 4096)
    T, al, al64 = oracle.quantise(W, with_alpha64=True)
    Wd = W.astype(np.float64)
    kept = np.where(T != 0, np.abs(Wd), 0.0).sum(1)
    lhs = np.array([err_of(W[i], T[i], al64[i]) for i in range(64)])
    rhs = (Wd ** 2).sum(1) - kept ** 2 / (0.75 * 4096)
    assert np.allclose(lhs, rhs, rtol=1e-10, atol=0)
    # fp32 alpha is the fp64 scale rounded once
    assert np.array_equal(al, al64.astype(np.float32))
    # kept weights are exactly the 3 largest |w| of each group (ties aside)
    g = np.abs(W).reshape(64, -1, 4)
    z = np.argmax((T.reshape(64, -1, 4) == 0), axis=2)
    assert np.all(np.take_along_axis(g, z[..., None], 2)[..., 0] <= g.min(2) + 0)


def test_quantise_tie_and_signed_zero_rules():
    W = np.array([[0.5, 0.5, 0.5, 0.5],      # all tied -> position 0 zeroed
                  [2.0, 1.0, 1.0, 3.0],      # tie between 1 and 2 -> 1 zeroed
                  [-0.0, 0.0, -1.0, 1.0],    # |-0| == |0| -> 0 zeroed; kept +0 is +1
                  [0.0, 0.0, 0.0, 0.0]],     # all zero row -> alpha 0, T = [0,1,1,1]
                 dtype=np.float32)
    T, al = oracle.quantise(W)
    assert T.tolist() == [[0, 1, 1, 1], [1, 0, 1, 1], [0, 1, -1, 1], [0, 1, 1, 1]]
    assert al[3] == 0.0


def test_quantise_rejects_nonfinite():
    W = np.ones((2, 8), dtype=np.float32)
    W[1, 3] = np.nan
    with pytest.raises(oracle.OracleError):
        oracle.quantise(W)


def test_page_example_block_golden():
    g = json.load(open(os.path.join(GOLDEN, "page_example_block.json")))
    W = np.array([g["w"]], dtype=np.float32)
    T, al = oracle.quantise(W)
    assert T[0].tolist() == g["T"]
    assert al[0] == np.float32(g["alpha"])
    code = oracle.encode_group(T[0])
    assert code == g["code"]
    p, s = oracle.code_to_pattern_sign(code)
    assert (p, s) == (g["pattern4"], g["sign_bit_from_page"])
    # 1.25 bit/weight: a row of K weights takes 5K/32 bytes
    for K in (32, 256, 4096, 14336):
        assert oracle.row_bytes(K) * 8 == K * g["bits_per_weight_from_page"]
    pats = {oracle.code_to_pattern_sign(c)[0] for c in range(32)}
    assert len(pats) == g["lut_entries_per_segment_from_page"]


# ------------------------------------------------------- codes and packing
def test_codes_exhaustive_three_nonzeros():
    seen = set()
    for c in range(32):
        t = oracle.decode_group(c)
        assert np.count_nonzero(t) == 3 and set(np.unique(t)) <= {-1, 0, 1}
        assert oracle.encode_group(t) == c
        seen.add(tuple(t.tolist()))
    assert seen == {tuple(v.tolist()) for v in all_34_patterns()}
    assert oracle.encode_group([1, 1, 1, 1]) == -1
    assert oracle.encode_group([0, 0, 1, 1]) == -1
    assert oracle.encode_group([2, 0, 1, 1]) == -1


def test_pattern_sign_bijection_and_meaning():
    pairs = set()
    for c in range(32):
        p, s = oracle.code_to_pattern_sign(c)
        assert 0 <= p < 16 and s in (0, 1)
        assert oracle.pattern_sign_to_code(p, s) == c
        pairs.add((p, s))
        base = oracle.decode_group(oracle.pattern_sign_to_code(p, 0))
        nz = base[base != 0]
        assert nz[0] == 1                        # table entries start with +1
        assert np.array_equal(oracle.decode_group(c), base * (-1 if s else 1))
    assert len(pairs) == 32


def _bits_of(row: np.ndarray, start: int, n: int) -> int:
    v = 0
    for b in range(n):
        bit = start + b
        v |= ((int(row[bit // 8]) >> (bit % 8)) & 1) << b
    return v


def test_pack_bit_positions_all_offsets():
    rng = np.random.default_rng(5)
    K = 64
    for code in range(32):
        for j in range(8):                       # 5j mod 8 covers every offset
            codes = rng.integers(0, 32, size=K // 4)
            codes[j] = code
            T = np.concatenate([oracle.decode_group(c) for c in codes])[None, :]
            packed = oracle.pack(T)
            assert packed.shape == (1, 10)
            assert _bits_of(packed[0], 5 * j, 5) == code
            for g in range(K // 4):
                assert _bits_of(packed[0], 5 * g, 5) == codes[g]
            assert np.array_equal(oracle.unpack(packed, K), T)


def test_random_streams_round_trip():
    rng = np.random.default_rng(6)
    for K in (32, 96, 256, 4096):
        raw = rng.integers(0, 256, size=(7, K * 5 // 32), dtype=np.uint8)
        T = oracle.unpack(raw, K)
        assert np.array_equal(oracle.pack(T), raw)      # every 5-bit value is a code
        assert np.all(np.count_nonzero(T.reshape(7, -1, 4), axis=2) == 3)


@pytest.mark.slow
def test_invariant_full_size_heavy_tail():
    """3 nonzeros in every group of the full K=8192, N=28672 stress weights."""
    W = synth.config_weights(4, 0, 8192, 28672)
    T, al = oracle.quantise(W)
    nz = np.count_nonzero(T.reshape(28672, -1, 4), axis=2)
    assert nz.min() == 3 and nz.max() == 3
    assert np.all(al > 0)
    codes = oracle.pack(T[:512])
    assert np.array_equal(oracle.unpack(codes, 8192), T[:512])


# ------------------------------------------------------------ contraction
@pytest.mark.parametrize("M,N,K", [(1, 128, 256), (3, 37, 96), (16, 64, 512), (5, 9, 4096)])
def test_gemm_vs_numpy_and_lut(M, N, K):
    rng = np.random.default_rng(M * 1000 + N)
    q = rng.integers(-127, 128, size=(M, K), dtype=np.int64).astype(np.int8)
    raw = rng.integers(0, 256, size=(N, K * 5 // 32), dtype=np.uint8)
    T = oracle.unpack(raw, K)
    ref = q.astype(np.int64) @ T.astype(np.int64).T
    acc = oracle.gemm(q, T)
    assert np.array_equal(acc, ref)
    assert np.array_equal(oracle.gemm_lut(q, raw, K), ref)


def test_gemm_extremes_no_overflow():
    K = 14336
    q = np.full((2, K), 127, dtype=np.int8)
    q[1] = -127
    T = oracle.unpack(np.zeros((1, K * 5 // 32), dtype=np.uint8), K)   # all +1 except z
    acc = oracle.gemm(q, T)
    assert acc[0, 0] == 127 * (3 * K // 4) and acc[1, 0] == -127 * (3 * K // 4)


# ------------------------------------------------------ activation quant
def test_quant_act_properties():
    x = synth.activations(4, 0, 8, 8192, outlier_frac=0.01, outlier_gain=20.0)
    q, s = oracle.quant_act(x)
    assert q.dtype == np.int8 and np.all(np.abs(q.astype(int)) <= 127)
    for m in range(8):
        k = np.argmax(np.abs(x[m]))
        assert abs(int(q[m, k])) == 127 and np.sign(q[m, k]) == np.sign(x[m, k])
        assert s[m] == np.float32(np.abs(x[m]).max() / np.float32(127.0))
        err = np.abs(x[m].astype(np.float64) - q[m].astype(np.float64) * float(s[m]))
        assert np.all(err <= 0.5 * float(s[m]) * (1 + 1e-6))


def test_quant_act_half_even_ties_and_zero_token():
    s = 0.125                                   # a = 127 * 2^-3 -> s = 2^-3 exactly
    j = np.arange(-126, 126)
    x = np.concatenate([[127 * s], (j + 0.5) * s]).astype(np.float32)[None, :]
    q, sc = oracle.quant_act(x)
    assert sc[0] == np.float32(s)
    half = q[0, 1:].astype(int)
    expect = np.where((j % 2) == 0, j, j + 1)   # round half to even
    assert np.array_equal(half, expect)
    z = np.zeros((2, 64), dtype=np.float32)
    qz, sz = oracle.quant_act(z)
    assert np.all(qz == 0) and np.all(sz == 0)


# --------------------------------------------------------------- epilogue
def test_epilogue_bounds_and_exact_cases():
    rng = np.random.default_rng(3)
    acc = rng.integers(-1_300_000, 1_300_000, size=(4, 300)).astype(np.int32)
    alpha = rng.uniform(0.001, 0.1, size=300).astype(np.float32)
    s = rng.uniform(0.001, 0.2, size=4).astype(np.float32)
    y = oracle.epilogue(acc, alpha, s)
    exact = acc.astype(np.float64) * alpha.astype(np.float64)[None] * s.astype(np.float64)[:, None]
    assert np.all(np.abs(y - exact) <= 2.0 ** -22 * np.abs(exact))
    a2 = (2.0 ** -rng.integers(3, 9, size=300)).astype(np.float32)
    s2 = (2.0 ** -rng.integers(2, 6, size=4)).astype(np.float32)
    y2 = oracle.epilogue(acc, a2, s2)
    assert np.array_equal(y2.astype(np.float64),
                          acc.astype(np.float64) * a2.astype(np.float64)[None] * s2.astype(np.float64)[:, None])


def test_forward_matches_pieces():
    W = synth.weights(0, 0, 128, 256)
    x = synth.activations(0, 0, 3, 256)
    y, acc, q, s, codes, alpha = oracle.reference(x, W)
    T = oracle.unpack(codes, 256)
    assert np.array_equal(acc, q.astype(np.int64) @ T.astype(np.int64).T)
    assert np.array_equal(y, oracle.epilogue(acc, alpha, s))
