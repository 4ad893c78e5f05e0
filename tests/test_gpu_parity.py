"""GPU parity: every step of the CUDA path against the oracle, through the C ABI.

Bar: int8 activations, scales and int32 accumulators bit-exact; fp32 outputs
within 1e-6 relative (they are expected bit-identical).  Small ragged shapes
are compared in full; the five workload configurations run at full size with
oracle rows sampled at tile edges and at random, plus a full comparison of
the accumulators with torch._int_mm (a library int8 GEMM) over the oracle's
ternary weights where its shape rules allow (M > 16)."""
import numpy as np
import pytest

import oracle
import sparse_bit_matmul_b200 as sbm
import synth
from sherry_testlib import assert_y_close, rows_sample, run_gpu, upload_weights

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sbm.load()
    assert sbm.last_device_status(reset=True) >= 0
    yield
    assert sbm.last_device_status() == 0


# ------------------------------------------------------------ quantiser
@pytest.mark.parametrize("M,K,cfg", [(1, 256, 0), (3, 4096, 1), (32, 14336, 2), (128, 8192, 4), (5, 32, 0)])
def test_quant_act_bitexact(M, K, cfg):
    x = synth.config_activations(cfg, 0, M, K)
    q_o, s_o = oracle.quant_act(x)
    q, s = sbm.quant_act(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_o)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_o.view(np.uint32))


def test_quant_act_ties_and_zero_rows():
    s = 0.125
    j = np.arange(-126, 126)
    row = np.concatenate([[127 * s], (j + 0.5) * s, np.zeros(32 - (1 + len(j)) % 32)]).astype(np.float32)
    x = np.stack([row, np.zeros_like(row), -row]).astype(np.float32)
    q_o, s_o = oracle.quant_act(x)
    q, sc = sbm.quant_act(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_o)
    assert np.array_equal(sc.cpu().numpy(), s_o)


@pytest.mark.parametrize("path", ["quant_act", "linear"])
def test_quant_near_rounding_boundaries(path):
    """Activations within a few ulp of the half-integer rounding boundaries of
    x / s (where a reciprocal-multiply shortcut could round the other way)
    and exactly on them: q must equal the oracle's IEEE-division result."""
    rng = np.random.default_rng(11)
    K = 4096
    rows = []
    for rel in (0.0, 1e-7, 3e-7, 1e-6, 4e-6, 2e-5, 4e-5, 1e-4):
        a = np.float32(rng.uniform(0.5, 8.0))
        s = np.float32(a / np.float32(127.0))
        k = rng.integers(-126, 126, size=K - 1).astype(np.float64)
        sign = rng.choice([-1.0, 1.0], size=K - 1)
        x = ((k + 0.5) * (1.0 + sign * rel) * np.float64(s)).astype(np.float32)
        x = np.clip(x, -a, a)
        rows.append(np.concatenate([[a], x]).astype(np.float32))
    x = np.stack(rows)
    q_o, s_o = oracle.quant_act(x)
    xd = torch.from_numpy(x).cuda()
    if path == "quant_act":
        q, sc = sbm.quant_act(xd)
    else:
        N = 256
        W = synth.weights(0, 9, N, K)
        native, alpha_d, _, _ = upload_weights(W)
        for m0 in range(0, x.shape[0], sbm.LINEAR_FUSED_MAX_M):        # fused launches only
            xs = xd[m0:m0 + sbm.LINEAR_FUSED_MAX_M].contiguous()
            qq = torch.empty(xs.shape, dtype=torch.int8, device="cuda")
            ss = torch.empty(xs.shape[0], dtype=torch.float32, device="cuda")
            acc = torch.empty((xs.shape[0], N), dtype=torch.int32, device="cuda")
            sbm.linear(xs, native, alpha_d, N, acc=acc, out_q=qq, out_s=ss)
            torch.cuda.synchronize()
            assert np.array_equal(qq.cpu().numpy(), q_o[m0:m0 + xs.shape[0]])
            assert np.array_equal(ss.cpu().numpy().view(np.uint32), s_o[m0:m0 + xs.shape[0]].view(np.uint32))
        return
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_o)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_o.view(np.uint32))


# --------------------------------------------------------------- repack
@pytest.mark.parametrize("N,K", [(300, 96), (128, 4096), (129, 224), (1, 32)])
def test_repack_layout(N, K):
    rng = np.random.default_rng(N + K)
    codes = rng.integers(0, 256, size=(N, K // 32 * 5), dtype=np.uint8)
    nat = sbm.repack(torch.from_numpy(codes).cuda(), N, K).cpu().numpy().view(np.uint32)
    Tn, Kc = -(-N // 128), -(-K // 128)
    assert nat.size == Tn * Kc * 5 * 128
    pad = np.zeros((Tn * 128, Kc * 20), dtype=np.uint8)
    pad[:N, :codes.shape[1]] = codes
    expect = pad.reshape(Tn, 128, Kc, 5, 4).view(np.uint32)[..., 0]      # [t][r][c][j]
    expect = expect.transpose(0, 2, 3, 1).copy()                        # [t][c][j][r]
    for j in range(5):                                                  # plane j: row r at (r + 8j) % 128
        expect[:, :, j, :] = np.roll(expect[:, :, j, :], 8 * j, axis=-1)
    expect = expect.reshape(-1)
    assert np.array_equal(nat, expect)


# ---------------------------------------------- small ragged shapes, full
SMALL = [(1, 128, 256), (1, 37, 96), (3, 300, 4096), (17, 129, 224), (33, 200, 512),
         (64, 256, 1024), (100, 130, 4096), (129, 257, 160), (256, 512, 2048), (7, 1, 32),
         (2, 4100, 1184), (4, 777, 14336), (1, 640, 9216), (2, 1, 32), (300, 1024, 2048),
         (200, 388, 4096), (130, 8192, 256), (8, 300, 2048), (16, 129, 4096), (32, 1000, 1024),
         (9, 77, 16384), (4, 333, 8192), (3, 200, 16384), (5, 50, 160), (24, 2000, 512),
         # whole tiles per CTA plus split tiles on a 148-SM grid: 149 tiles
         # of one chunk (one split unit), 150 tiles of five chunks (split
         # units fewer than CTAs), 200 tiles of eight chunks (split units
         # shared out by floor division)
         (100, 19072, 128), (300, 6400, 640), (520, 5120, 1024),
         # fewer tiles than SMs with long K: every tile split into equal K
         # shares over many CTAs (128- and 64-token tiles)
         (130, 384, 14336), (40, 256, 14336),
         # 192-token tiles (M >= 1536), the last one ragged
         (1600, 300, 512),
         # one token with rows longer than the fused quantiser holds in
         # registers (K / 4 > 7 float4s per thread): x streams from memory
         (1, 300, 16384), (1, 4100, 16384)]


def _kernel_serves(kernel: str, M: int, K: int) -> bool:
    if kernel == "gemv":
        return M <= sbm.GEMV_MAX_M and K <= 16384
    if kernel == "decode":
        return M <= sbm.DECODE_MAX_M
    return True


@pytest.mark.parametrize("kernel", ["auto", "linear", "decode", "tc", "gemv", "simt"])
@pytest.mark.parametrize("M,N,K", SMALL)
def test_gemm_small_full(M, N, K, kernel):
    if not _kernel_serves(kernel, M, K):
        pytest.skip(f"the {kernel} kernel does not serve M={M}, K={K}")
    W = synth.weights(0, 1, N, K, sigma=0.02)
    x = synth.activations(0, 1, M, K)
    y_o, acc_o, q_o, s_o, codes_o, alpha_o = oracle.reference(x, W)
    native, alpha_d, codes, alpha = upload_weights(W)
    assert np.array_equal(codes, codes_o) and np.array_equal(alpha, alpha_o)
    y, acc, q, s = run_gpu(x, native, alpha_d, N, kernel)
    assert np.array_equal(q, q_o) and np.array_equal(s, s_o)
    assert np.array_equal(acc, acc_o)
    assert_y_close(y, y_o)
    if kernel in ("auto", "tc", "linear"):
        y2, _, _, _ = run_gpu(x, native, alpha_d, N, kernel, with_acc=False)
        assert np.array_equal(y2, y)


def test_gemm_zero_token_and_repeat():
    """all-zero token -> y = 0; repeated calls agree (workspace left clean)."""
    N, K = 300, 1024
    W = synth.weights(0, 2, N, K)
    x = synth.activations(0, 2, 5, K)
    x[2] = 0.0
    native, alpha_d, _, _ = upload_weights(W)
    first = run_gpu(x, native, alpha_d, N)
    assert np.all(first[0][2] == 0) and np.all(first[1][2] == 0)
    for _ in range(3):
        again = run_gpu(x, native, alpha_d, N)
        assert np.array_equal(again[1], first[1]) and np.array_equal(again[0], first[0])
    y_o, acc_o, *_ = oracle.reference(x, W)
    assert np.array_equal(first[1], acc_o)


# ----------------------------------------------- full-size configurations
def _full_size_check(cfg, copy, M_list, K, N, int_mm=True, kernels=("auto",)):
    """One workload configuration at full size.  The codes and alpha of every
    row are compared with the oracle's.  For M <= 16 the oracle computes
    every output, and the whole int32 acc (bit-exact) and y (1e-6 relative)
    are compared.  Larger M compares oracle rows sampled at tile edges and at
    random, and every accumulator against torch._int_mm over the oracle's
    ternary weights."""
    W = synth.config_weights(cfg, copy, K, N)
    native, alpha_d, codes, alpha = upload_weights(W)
    T_full, a_full = oracle.quantise(W)
    assert np.array_equal(codes, oracle.pack(T_full))
    assert np.array_equal(alpha, a_full)
    rows = rows_sample(N, seed=cfg * 7 + N)
    for M in M_list:
        x = synth.config_activations(cfg, copy, M, K)
        q_o, s_o = oracle.quant_act(x)
        cols = np.arange(N) if M <= 16 else rows
        acc_o = oracle.gemm(q_o, T_full if M <= 16 else T_full[rows])
        y_o = oracle.epilogue(acc_o, a_full[cols], s_o)
        for kern in kernels:
            if not _kernel_serves(kern, M, K):
                continue
            y, acc, q, s = run_gpu(x, native, alpha_d, N, kern)
            assert np.array_equal(q, q_o) and np.array_equal(s, s_o)
            assert np.array_equal(acc[:, cols], acc_o), kern
            assert_y_close(y[:, cols], y_o)
            y2, _, _, _ = run_gpu(x, native, alpha_d, N, kern, with_acc=False)
            assert np.array_equal(y2, y), kern          # y-only path (TMA stores) gives the same y
        if int_mm and M > 16:
            ref = torch._int_mm(torch.from_numpy(q_o).cuda(), torch.from_numpy(T_full).cuda().t().contiguous())
            assert torch.equal(torch.from_numpy(acc).cuda(), ref)
    return W


@pytest.mark.parametrize("K,N", synth.PROJ_SHAPES)
def test_config1_decode_full_size(K, N):
    _full_size_check(1, 0, [1], K, N, kernels=("auto", "linear", "decode", "tc", "gemv"))


@pytest.mark.parametrize("K,N", synth.PROJ_SHAPES)
def test_config2_small_batch_full_size(K, N):
    _full_size_check(2, 0, [4, 8, 16, 32], K, N, kernels=("auto", "linear", "decode", "tc"))


@pytest.mark.parametrize("K,N", [(4096, 14336), (14336, 4096)])
def test_config3_prefill_full_size(K, N):
    _full_size_check(3, 0, [2048], K, N)


def test_config4_heavy_tail_full_size():
    W = _full_size_check(4, 0, [1, 128, 4096], 8192, 28672, kernels=("auto", "linear", "decode", "tc"))
    T, _ = oracle.quantise(W)
    assert np.all(np.count_nonzero(T.reshape(28672, -1, 4), axis=2) == 3)


@pytest.mark.parametrize("M,N,K,kernel", [(1, 256, 14336, "decode"), (2, 256, 14336, "decode"),
                                          (1, 256, 14336, "linear"), (1, 256, 14336, "gemv"),
                                          (4, 256, 14336, "tc"), (16, 256, 14336, "tc"),
                                          (4, 256, 14336, "gemv"), (8, 256, 4096, "decode"),
                                          (130, 512, 14336, "tc")])
def test_accumulator_extremes(M, N, K, kernel):
    """The largest sums the method can form: every activation quantises to
    +127 or -127 and every row is all +1 or all -1 on its kept weights, so
    |acc| = 127 * 0.75 K (1,365,504 at K = 14336).  Through the decode
    kernel, the fused linear path, the table GEMV and the tensor cores (the
    small-M shapes split every tile's K range over many CTAs, whose int32
    partial sums meet in the workspace)."""
    # groups of 4 positive weights with distinct magnitudes: position 0 is
    # zeroed, 1..3 keep +1; the second half of the rows is negated
    g = np.array([1.0, 2.0, 3.0, 4.0], dtype=np.float32) * 0.01
    W = np.tile(g, (N, K // 4))
    W[N // 2:] *= -1.0
    x = np.ones((M, K), dtype=np.float32)
    x[1::2] *= -1.0                                     # odd tokens: every activation -127
    y_o, acc_o, q_o, s_o, codes_o, alpha_o = oracle.reference(x, W)
    assert np.all(np.abs(q_o) == 127)
    full = 127 * 3 * (K // 4)
    assert np.all(np.abs(acc_o) == full)
    native, alpha_d, codes, alpha = upload_weights(W)
    assert np.array_equal(codes, codes_o)
    y, acc, q, s = run_gpu(x, native, alpha_d, N, kernel)
    assert np.array_equal(acc, acc_o)
    assert_y_close(y, y_o)


def test_config0_tiny_exact():
    W = synth.config_weights(0, 0, 256, 128)
    x = synth.config_activations(0, 0, 1, 256)
    y_o, acc_o, *_ = oracle.reference(x, W)
    native, alpha_d, _, _ = upload_weights(W)
    for kernel in ("auto", "linear", "decode", "tc", "gemv", "simt"):
        y, acc, _, _ = run_gpu(x, native, alpha_d, 128, kernel)
        assert np.array_equal(acc, acc_o)
        assert np.array_equal(y, y_o)


# ------------------------------------------------- layers chained on one stream
@pytest.mark.parametrize("route", ["linear", "quant+gemm", "quant+tc"])
@pytest.mark.parametrize("M", [1, 2, 8, 64])
def test_chained_layers_one_stream(M, route):
    """Six layers, each fed the previous layer's output, queued on one stream
    with no synchronisation in between: the kernels start early under
    programmatic dependent launch, so a read of the activations before the
    previous layer finished would show here.  Each layer must equal the
    oracle applied to the device's own previous output."""
    K = N = 1024
    L = 6
    Ws = [synth.weights(7, i, N, K) for i in range(L)]
    ups = [upload_weights(W) for W in Ws]
    x0 = synth.activations(7, 0, M, K)
    xd = torch.from_numpy(x0).cuda()
    ys, accs = [], []
    cur = xd
    for i, (native, alpha_d, _, _) in enumerate(ups):
        y = torch.empty((M, N), dtype=torch.float32, device="cuda")
        acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
        if route == "linear":
            sbm.linear(cur, native, alpha_d, N, out=y, acc=acc)
        else:
            q, s = sbm.quant_act(cur)
            sbm.gemm(q, s, native, alpha_d, N, out=y, acc=acc, kernel="tc" if route == "quant+tc" else "auto")
        ys.append(y)
        accs.append(acc)
        cur = y
    torch.cuda.synchronize()
    prev = x0
    for i in range(L):
        y_o, acc_o, *_ = oracle.reference(prev, Ws[i])
        assert np.array_equal(accs[i].cpu().numpy(), acc_o), f"layer {i}"
        y_i = ys[i].cpu().numpy()
        assert_y_close(y_i, y_o)
        prev = y_i
