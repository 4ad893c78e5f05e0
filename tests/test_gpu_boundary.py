"""The C ABI's contract on the device: the asynchronous entry points allocate
no memory, a call that needs more workspace than was reserved is refused
before anything is launched, and failure detection works end to end (a
bounded wait that runs out is reported through the device status word and
the context stays usable)."""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest

import oracle
import sparse_bit_matmul_b200 as sbm
import synth
from sherry_testlib import assert_y_close, upload_weights

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sbm.load()
    assert sbm.last_device_status(reset=True) >= 0
    yield
    assert sbm.last_device_status() == 0


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_async_calls_allocate_nothing():
    """After sherry_reserve, first calls on fresh shapes of every asynchronous
    entry point family (decode kernel, fused linear, tensor cores with split
    tiles, two-launch linear, W4A8) leave the device's free memory unchanged.
    Run in a child process with CUDA_MODULE_LOADING=EAGER: with lazy loading
    the driver takes device memory for a kernel's code at its first launch,
    which would hide or mimic an allocation by the library."""
    env = dict(os.environ, CUDA_MODULE_LOADING="EAGER")
    res = subprocess.run([sys.executable, os.path.join(HERE, "async_alloc_check.py")], env=env,
                         capture_output=True, text=True, timeout=600)
    assert res.returncode == 0 and res.stdout.strip().endswith("ok"), res.stdout + res.stderr


def test_call_beyond_reservation_is_refused():
    """A tensor-core launch with split tiles and a token tile larger than any
    reserved so far returns SHERRY_ERR_WORKSPACE without launching."""
    L = sbm.load()
    M, N, K = 4000, 1024, 256      # 192-token tiles: 168 tiles on 148 SMs, 20 of them split
    reserved = sbm._reserved.get(torch.cuda.current_device(), (0, 0))[0]
    if reserved >= 1536:
        pytest.skip("a 192-token workspace is already reserved in this process")
    W = synth.weights(8, 99, N, K)
    native, alpha, _, _ = upload_weights(W)
    q = torch.ones((M, K), dtype=torch.int8, device="cuda")
    s = torch.ones(M, dtype=torch.float32, device="cuda")
    y = torch.full((M, N), 7.0, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    rc = L.sherry_gemm(q.data_ptr(), s.data_ptr(), native.data_ptr(), alpha.data_ptr(), y.data_ptr(), M, N, K,
                       _stream())
    assert rc == sbm.ERR_WORKSPACE, sbm.status_string(rc)
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)                       # nothing ran
    sbm.reserve(M, K)
    y = sbm.gemm(q, s, native, alpha, N)
    torch.cuda.synchronize()
    T, a = oracle.quantise(W)
    acc_o = oracle.gemm(q.cpu().numpy(), T)
    assert_y_close(y.cpu().numpy(), oracle.epilogue(acc_o, a, s.cpu().numpy()))


def test_bounded_wait_runs_out_and_is_reported():
    """sherry_selftest_wait waits 1 ms for an mbarrier phase nothing
    completes: the kernel returns, the status word holds the self-test code,
    a reset clears it, and the context keeps working (a GEMM afterwards
    matches the oracle)."""
    assert sbm.last_device_status(reset=True) == 0
    sbm.selftest_wait(1_000_000)
    torch.cuda.synchronize()
    assert sbm.last_device_status() == sbm.DEV_TIMEOUT_SELFTEST
    assert sbm.last_device_status(reset=True) == sbm.DEV_TIMEOUT_SELFTEST
    assert sbm.last_device_status() == 0
    M, N, K = 5, 300, 1024
    W = synth.weights(8, 7, N, K)
    x = synth.activations(8, 7, M, K)
    native, alpha, _, _ = upload_weights(W)
    q, s = sbm.quant_act(torch.from_numpy(x).cuda())
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    sbm.gemm(q, s, native, alpha, N, acc=acc, kernel="tc")
    torch.cuda.synchronize()
    _, acc_o, *_ = oracle.reference(x, W)
    assert np.array_equal(acc.cpu().numpy(), acc_o)
    assert sbm.last_device_status() == 0


def test_selftest_rejects_bad_limits():
    L = sbm.load()
    assert L.sherry_selftest_wait(0, None) == sbm.ERR_INVALID_ARG
    assert L.sherry_selftest_wait(2_000_000_000, None) == sbm.ERR_INVALID_ARG
