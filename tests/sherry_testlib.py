"""Helpers shared by the GPU tests: seeded problems, device upload through the
public binding, and oracle values for sampled rows."""
from __future__ import annotations

import numpy as np

import oracle
import sparse_bit_matmul_b200 as sbm
import synth


def rows_sample(N: int, count: int = 48, seed: int = 0) -> np.ndarray:
    """Rows at tile edges plus random rows."""
    rng = np.random.default_rng(seed)
    edges = {0, 1, 127, 128, N - 1, N - 2, N // 2, (N // 128) * 128 - 1}
    edges = {e for e in edges if 0 <= e < N}
    rest = rng.choice(N, size=min(N, count), replace=False)
    return np.array(sorted(edges | set(rest.tolist())), dtype=np.int64)


def upload_weights(W: np.ndarray, device="cuda"):
    """Host pack (product) -> device -> repack; returns (native, alpha_dev, codes)."""
    import torch
    codes, alpha = sbm.pack(W)
    N, K = W.shape
    native = sbm.repack(torch.from_numpy(codes).to(device), N, K)
    return native, torch.from_numpy(alpha).to(device), codes, alpha


def run_gpu(x: np.ndarray, native, alpha_dev, N: int, kernel="auto", with_acc: bool = True):
    """quant_act + gemm on the device (kernel "linear": sherry_linear from the
    fp32 activations); returns numpy (y, acc, q, s).

    with_acc=False asks for y only -- the configuration of the benchmark,
    where the tensor-core kernel writes complete output tiles with TMA
    stores -- and returns acc = None."""
    import torch
    xd = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    M = x.shape[0]
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda") if with_acc else None
    if kernel == "linear":
        # fp32 activations straight in (sherry_linear / sherry_linear_ex)
        if with_acc:
            q = torch.empty((M, x.shape[1]), dtype=torch.int8, device="cuda")
            s = torch.empty(M, dtype=torch.float32, device="cuda")
            y = sbm.linear(xd, native, alpha_dev, N, acc=acc, out_q=q, out_s=s)
        else:
            y = sbm.linear(xd, native, alpha_dev, N)
            q, s = sbm.quant_act(xd)
    else:
        q, s = sbm.quant_act(xd)
        y = sbm.gemm(q, s, native, alpha_dev, N, acc=acc, kernel=kernel)
    torch.cuda.synchronize()
    if acc is None:
        return y.cpu().numpy(), None, q.cpu().numpy(), s.cpu().numpy()
    return y.cpu().numpy(), acc.cpu().numpy(), q.cpu().numpy(), s.cpu().numpy()


def assert_y_close(y_gpu: np.ndarray, y_ref: np.ndarray, rtol: float = 1e-6):
    """fp32 outputs: within rtol relative (they are expected bit-identical:
    the same two fp32 products in the same order on exact integers)."""
    diff = np.abs(y_gpu.astype(np.float64) - y_ref.astype(np.float64))
    bound = rtol * np.abs(y_ref.astype(np.float64)) + 1e-30
    bad = diff > bound
    assert not bad.any(), f"{bad.sum()} outputs beyond {rtol} relative; first at {np.argwhere(bad)[0]}"
