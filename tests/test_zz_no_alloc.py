"""sherry_gemm_noalloc: the GEMM entry point for callers that cannot allocate
device memory while they run (their memory comes from a pool sized at
start-up, or their request loop may not make synchronising cudaMalloc /
cudaFree calls).  It keeps its split-K scratch in a fixed array inside the
library instead of a workspace allocated on first use.

Checked through the C ABI against sherry_gemm_acc (the entry point with the
allocated workspace) on two calls in a row: int32 accumulators bit-exact,
fp32 outputs within 1e-6 relative.  Kept in a file of its own that pytest
collects last; it passes alone in a fresh process and after the others."""
import ctypes

import numpy as np
import pytest

import sparse_bit_matmul_b200 as sbm
import synth
from sherry_testlib import assert_y_close, upload_weights

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# (M, N, K): decode sizes, one shape whose tiles are split over many CTAs
CASES = [(1, 4096, 4096), (7, 300, 4096), (32, 1000, 1024), (16, 128, 256)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sbm.load()


def _call(entry, q, s, native, alpha, N):
    M, K = q.shape
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    L = sbm.load()
    rc = getattr(L, entry)(q.data_ptr(), s.data_ptr(), native.data_ptr(), alpha.data_ptr(), y.data_ptr(),
                           acc.data_ptr(), M, N, K,
                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == sbm.OK, sbm.status_string(rc)
    torch.cuda.synchronize()
    return y.cpu().numpy(), acc.cpu().numpy()


@pytest.mark.parametrize("M,N,K", CASES)
def test_noalloc_matches_gemm_acc_two_calls(M, N, K):
    W = synth.weights(5, M, N, K)
    x = synth.activations(5, M, M, K)
    native, alpha, _, _ = upload_weights(W)
    q, s = sbm.quant_act(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    first = _call("sherry_gemm_noalloc", q, s, native, alpha, N)
    second = _call("sherry_gemm_noalloc", q, s, native, alpha, N)
    assert torch.cuda.mem_get_info()[0] == free_before      # nothing allocated
    y_ref, acc_ref = _call("sherry_gemm_acc", q, s, native, alpha, N)
    for y, acc in (first, second):
        assert np.array_equal(acc, acc_ref)
        assert_y_close(y, y_ref, rtol=1e-6)
    assert sbm.last_device_status() == 0


def test_noalloc_rejects_more_than_32_tokens():
    L = sbm.load()
    dummy = torch.zeros(64 * 256, dtype=torch.int8, device="cuda")
    p = dummy.data_ptr()
    rc = L.sherry_gemm_noalloc(p, p, p, p, p, None, 33, 128, 256, None)
    assert rc == sbm.ERR_UNSUPPORTED_SHAPE
