"""GPU parity of the W4A8 FastGEMM path (OdysseyLLM review page,
xllm-io.github.io/paper-review/blog/odysseyllm, sec. 3.1-3.3, 5.2) against
the oracle, through the C ABI.

Bar: the int32 sums (after the division by 16) bit-exact; fp32 outputs within
1e-6 relative (they are expected bit-identical: the same two fp32 products
in the same order on exact integers).  Small ragged shapes are compared in
full; the prefill and decode shapes run at full size with oracle rows sampled
at tile edges and at random, plus a full comparison of the sums with
torch._int_mm (a library int8 GEMM) over the oracle's int4 weights where its
shape rules allow (M > 16)."""
import numpy as np
import pytest

import oracle
import sparse_bit_matmul_b200 as sbm
import synth
from sherry_testlib import assert_y_close, rows_sample

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


def upload_w4(W: np.ndarray):
    """Host pack (product) -> device -> repack; returns (native, scale_dev, w4, scale)."""
    w4, scale = sbm.w4a8_pack(W)
    N, K = W.shape
    native = sbm.w4a8_repack(torch.from_numpy(w4).cuda(), N, K)
    return native, torch.from_numpy(scale).cuda(), w4, scale


def run_w4(x: np.ndarray, native, scale_d, N: int, with_acc: bool = True, kernel: str = "auto"):
    xd = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    M = x.shape[0]
    q, s = sbm.quant_act(xd)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda") if with_acc else None
    y = sbm.w4a8_gemm(q, s, native, scale_d, N, acc=acc, kernel=kernel)
    torch.cuda.synchronize()
    return (y.cpu().numpy(), acc.cpu().numpy() if with_acc else None, q.cpu().numpy(), s.cpu().numpy())


@pytest.mark.parametrize("N,K", [(300, 96), (128, 4096), (129, 224), (1, 32)])
def test_w4a8_repack_layout(N, K):
    rng = np.random.default_rng(N * 7 + K)
    Wq = rng.integers(-8, 8, size=(N, K)).astype(np.int64)
    w4 = oracle.w4a8_pack(Wq.astype(np.int8))
    nat = sbm.w4a8_repack(torch.from_numpy(w4).cuda(), N, K).cpu().numpy()
    Tn, Kc = -(-N // 128), -(-K // 128)
    pad = np.zeros((Tn * 128, Kc * 128), dtype=np.int64)
    pad[:N, :K] = Wq
    # k = 128 c + 32 q + 8 i + 4 h + b; byte (q, i, b) = w[h=0] & 15 | (w[h=1] & 15) << 4
    v = pad.reshape(Tn, 128, Kc, 4, 4, 2, 4) & 15
    byte = (v[:, :, :, :, :, 0, :] | (v[:, :, :, :, :, 1, :] << 4)).astype(np.uint8)   # [t][r][c][q][i][b]
    expect = byte.transpose(0, 2, 3, 1, 4, 5).reshape(-1)                                 # [t][c][q][r][i][b]
    assert np.array_equal(nat, expect)


SMALL = [(1, 128, 256), (1, 37, 96), (3, 300, 4096), (17, 129, 224), (33, 200, 512),
         (64, 256, 1024), (100, 130, 4096), (129, 257, 160), (7, 1, 32), (2, 4100, 1184),
         (4, 777, 14336), (16, 129, 4096), (32, 1000, 1024), (9, 77, 16384), (300, 1024, 2048),
         # whole tiles plus split tiles on a 148-SM grid; fewer tiles than SMs
         # with long K (every tile split into K shares)
         (100, 19072, 128), (130, 384, 14336), (40, 256, 14336),
         # 192-token tiles (M >= 1536), the last one ragged
         (1600, 300, 512)]


@pytest.mark.parametrize("kernel", ["auto", "tc", "gemv"])
@pytest.mark.parametrize("M,N,K", SMALL)
def test_w4a8_small_full(M, N, K, kernel):
    if kernel == "gemv" and M > sbm.W4A8_GEMV_MAX_M:
        pytest.skip("the GEMV serves M <= 4")
    W = synth.weights(0, 3, N, K, sigma=0.02)
    x = synth.activations(0, 3, M, K)
    y_o, acc_o, q_o, s_o, w4_o, S_o = oracle.w4a8_reference(x, W)
    native, scale_d, w4, scale = upload_w4(W)
    assert np.array_equal(w4, w4_o) and np.array_equal(scale, S_o)
    y, acc, q, s = run_w4(x, native, scale_d, N, kernel=kernel)
    assert np.array_equal(q, q_o) and np.array_equal(s, s_o)
    assert np.array_equal(acc, acc_o)
    assert_y_close(y, y_o)
    y2, _, _, _ = run_w4(x, native, scale_d, N, with_acc=False, kernel=kernel)   # y only (TMA stores on tc)
    assert np.array_equal(y2, y)


@pytest.mark.parametrize("M,kernel", [(3, "gemv"), (3, "auto"), (20, "auto")])
def test_w4a8_extreme_values_near_int32(M, kernel):
    """w = -8 (bit pattern 1000, not produced by the quantiser) and q = +-127
    at K = 14336: the x16 sums reach -127 * 128 * K = -2.3e8, on the CUDA-core
    GEMV and on the tensor-core kernel."""
    N, K = 256, 14336
    w4 = np.full((N, K // 2), 0x88, dtype=np.uint8)            # every weight -8
    w4[1::2] = 0x77                                             # odd rows: +7
    native = sbm.w4a8_repack(torch.from_numpy(w4).cuda(), N, K)
    scale_d = torch.full((N,), 0.5, dtype=torch.float32, device="cuda")
    x = np.ones((M, K), dtype=np.float32)
    x[1::2] = -1.0
    q_o, s_o = oracle.quant_act(x)
    acc_o = oracle.w4a8_gemm(q_o, w4, K)
    assert acc_o[0, 0] == -8 * 127 * K and acc_o[1, 1] == -7 * 127 * K
    xd = torch.from_numpy(x).cuda()
    q, s = sbm.quant_act(xd)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    y = sbm.w4a8_gemm(q, s, native, scale_d, N, acc=acc, kernel=kernel)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy(), acc_o)
    assert_y_close(y.cpu().numpy(), oracle.w4a8_epilogue(acc_o, np.full(N, 0.5, np.float32), s_o))


@pytest.mark.parametrize("M,kernel", [(3, "gemv"), (3, "auto"), (5, "auto")])
def test_w4a8_zero_token_and_repeat(M, kernel):
    N, K = 300, 1024
    W = synth.weights(0, 4, N, K)
    x = synth.activations(0, 4, M, K)
    x[2] = 0.0
    native, scale_d, _, _ = upload_w4(W)
    first = run_w4(x, native, scale_d, N, kernel=kernel)
    assert np.all(first[0][2] == 0) and np.all(first[1][2] == 0)
    for _ in range(3):
        again = run_w4(x, native, scale_d, N, kernel=kernel)
        assert np.array_equal(again[1], first[1]) and np.array_equal(again[0], first[0])


@pytest.mark.parametrize("M,K,N,kernel", [(1, 4096, 14336, "auto"), (1, 4096, 14336, "gemv"),
                                          (4, 14336, 4096, "auto"), (4, 14336, 4096, "gemv"),
                                          (8, 14336, 4096, "auto"), (2048, 4096, 14336, "auto"),
                                          (2048, 14336, 4096, "auto")])
def test_w4a8_full_size_sampled(M, K, N, kernel):
    """Full-size shapes.  Up to 16 tokens the oracle computes every output:
    packing, int32 sums and y are compared over the whole matrix.  Above
    that, oracle rows sampled at tile edges and at random, plus every sum
    against torch._int_mm over the oracle's int4 weights."""
    cfg = 1 if M == 1 else (2 if M <= 32 else 3)
    W = synth.config_weights(cfg, 0, K, N)
    native, scale_d, w4, scale = upload_w4(W)
    x = synth.config_activations(cfg, 0, M, K)
    q_o, s_o = oracle.quant_act(x)
    if M <= 16:
        rows = np.arange(N)
        Wq_rows, S_rows = oracle.w4a8_quantise(W)
    else:
        rows = rows_sample(N, seed=M + N)
        Wq_rows, S_rows = oracle.w4a8_quantise(W[rows])
    packed_rows = oracle.w4a8_pack(Wq_rows)
    assert np.array_equal(w4[rows], packed_rows) and np.array_equal(scale[rows], S_rows)
    acc_o = oracle.w4a8_gemm(q_o, packed_rows, K)
    y, acc, q, s = run_w4(x, native, scale_d, N, kernel=kernel)
    assert np.array_equal(q, q_o) and np.array_equal(s, s_o)
    assert np.array_equal(acc[:, rows], acc_o)
    assert_y_close(y[:, rows], oracle.w4a8_epilogue(acc_o, S_rows, s_o))
    y2, _, _, _ = run_w4(x, native, scale_d, N, with_acc=False, kernel=kernel)
    assert np.array_equal(y2, y)
    if M > 16:
        Wq_full = oracle.w4a8_unpack(w4, K)
        ref = torch._int_mm(torch.from_numpy(q_o).cuda(), torch.from_numpy(Wq_full).cuda().t().contiguous())
        assert torch.equal(torch.from_numpy(acc).cuda(), ref)


def test_w4a8_linear_layer_object():
    """W4A8Linear: host pack, device repack, quantiser + GEMM in forward()."""
    N, K, M = 200, 1024, 3
    W = synth.weights(0, 6, N, K)
    x = synth.activations(0, 6, M, K)
    y_o, *_ = oracle.w4a8_reference(x, W)
    layer = sbm.W4A8Linear.from_weights(W, device="cuda")
    y = layer.forward(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    assert_y_close(y.cpu().numpy(), y_o)
