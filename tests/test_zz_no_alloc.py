"""sherry_gemm_noalloc: the GEMM entry point for callers that cannot allocate
device memory while they run (their memory comes from a pool sized at
start-up, or their request loop may not make synchronising cudaMalloc /
cudaFree calls).  It keeps its split-K scratch in a fixed array inside the
library instead of a workspace set aside by the caller or by sherry_reserve.

Checked through the C ABI on two calls in a row against the oracle (int32
accumulators bit-exact, fp32 outputs within 1e-6 relative) and against
sherry_gemm_acc, the entry point with the reserved workspace.  The shapes
cover the decode kernel (no scratch), tiles split over many CTAs, more row
tiles than SMs (whole tiles plus split leftovers, where scratch slots and
counters are reused), and y-only calls (acc = NULL) whose complete tiles
leave through TMA stores.  Kept in a file of its own that pytest collects
last; it passes alone in a fresh process and after the others."""
import ctypes

import numpy as np
import pytest

import oracle
import sparse_bit_matmul_b200 as sbm
import synth
from sherry_testlib import assert_y_close, upload_weights

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# (M, N, K, with_acc)
CASES = [(1, 4096, 4096, True), (7, 300, 4096, True), (32, 1000, 1024, True), (16, 128, 256, True),
         (16, 28672, 8192, True), (32, 19072, 4096, True),
         (7, 4096, 4096, False), (32, 4096, 4096, False), (16, 28672, 8192, False)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sbm.load()


def _call(entry, q, s, native, alpha, N, with_acc=True):
    M, K = q.shape
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda") if with_acc else None
    L = sbm.load()
    rc = getattr(L, entry)(q.data_ptr(), s.data_ptr(), native.data_ptr(), alpha.data_ptr(), y.data_ptr(),
                           acc.data_ptr() if with_acc else None, M, N, K,
                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == sbm.OK, sbm.status_string(rc)
    torch.cuda.synchronize()
    return y.cpu().numpy(), (acc.cpu().numpy() if with_acc else None)


@pytest.mark.parametrize("M,N,K,with_acc", CASES)
def test_noalloc_matches_oracle_two_calls(M, N, K, with_acc):
    W = synth.weights(5, M, N, K)
    x = synth.activations(5, M, M, K)
    native, alpha, _, _ = upload_weights(W)
    q, s = sbm.quant_act(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    y_o, acc_o, q_o, s_o, _, _ = oracle.reference(x, W)
    assert np.array_equal(q.cpu().numpy(), q_o)
    sbm.reserve(M, N, K)                                    # the reference entry point's workspace
    free_before = torch.cuda.mem_get_info()[0]
    first = _call("sherry_gemm_noalloc", q, s, native, alpha, N, with_acc)
    second = _call("sherry_gemm_noalloc", q, s, native, alpha, N, with_acc)
    assert torch.cuda.mem_get_info()[0] == free_before      # nothing allocated
    y_ref, acc_ref = _call("sherry_gemm_acc", q, s, native, alpha, N, with_acc)
    for y, acc in (first, second):
        if with_acc:
            assert np.array_equal(acc, acc_o)
            assert np.array_equal(acc, acc_ref)
        assert_y_close(y, y_o, rtol=1e-6)
        assert_y_close(y, y_ref, rtol=1e-6)
    assert sbm.last_device_status() == 0


def test_noalloc_rejects_more_than_32_tokens():
    L = sbm.load()
    dummy = torch.zeros(64 * 256, dtype=torch.int8, device="cuda")
    p = dummy.data_ptr()
    rc = L.sherry_gemm_noalloc(p, p, p, p, p, None, 33, 128, 256, None)
    assert rc == sbm.ERR_UNSUPPORTED_SHAPE
