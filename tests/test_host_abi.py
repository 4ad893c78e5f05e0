"""Host half of the C ABI (no GPU): the library loads, exports every entry
point declared in include/sherry.h, and the host packer/unpacker equal the
oracle byte for byte (Sherry page sec. 2.1 / 3.1)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import sparse_bit_matmul_b200 as sbm
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "sherry.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sherry_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_header_symbol(lib):
    names = header_functions()
    assert len(names) >= 12
    so = ctypes.CDLL(sbm.SO_PATH)
    for n in names:
        assert hasattr(so, n), f"{n} declared in sherry.h but not exported"
    assert set(names) == set(sbm.ABI_SYMBOLS)


def test_sizes_and_status(lib):
    assert sbm.packed_bytes(4096, 4096) == 4096 * 4096 * 5 // 32
    assert sbm.packed_bytes(128, 96) == 128 * 15
    assert sbm.packed_bytes(10, 100) == 0          # K % 32 != 0
    assert sbm.native_bytes(128, 256) == 1 * 2 * 2560
    assert sbm.native_bytes(129, 4096) == 2 * 32 * 2560
    assert sbm.native_bytes(4096, 14336) == 32 * 112 * 2560
    for s in range(6):
        assert sbm.status_string(s)
    assert lib.load().sherry_version() >= 10000


@pytest.mark.parametrize("N,K,cfg", [(128, 256, 0), (37, 96, 0), (300, 4096, 1), (64, 8192, 4)])
def test_pack_equals_oracle(N, K, cfg, lib):
    W = synth.config_weights(cfg, 0, K, N)
    codes, alpha = sbm.pack(W)
    T, a_o = oracle.quantise(W)
    assert np.array_equal(codes, oracle.pack(T))
    assert np.array_equal(alpha.view(np.uint32), a_o.view(np.uint32))
    assert np.array_equal(sbm.unpack(codes, K), T)


def test_pack_edge_rows(lib):
    W = np.zeros((6, 32), dtype=np.float32)
    W[1] = 0.5                                     # all ties
    W[2, :4] = [-0.0, 0.0, -1.0, 1.0]              # signed zeros
    W[3] = -np.arange(32, dtype=np.float32)        # descending magnitudes, negative
    W[4] = np.float32(1e-38)                       # tiny equal values
    W[5, ::2] = 3.0
    codes, alpha = sbm.pack(W)
    T, a_o = oracle.quantise(W)
    assert np.array_equal(codes, oracle.pack(T))
    assert np.array_equal(alpha, a_o)


def test_unpack_any_stream(lib):
    rng = np.random.default_rng(11)
    raw = rng.integers(0, 256, size=(9, 160), dtype=np.uint8)
    assert np.array_equal(sbm.unpack(raw, 1024), oracle.unpack(raw, 1024))


def test_argument_errors(lib):
    L = lib.load()
    W = np.ones((4, 32), dtype=np.float32)
    codes = np.empty((4, 5), dtype=np.uint8)
    alpha = np.empty(4, dtype=np.float32)
    assert L.sherry_pack(None, 4, 32, codes.ctypes.data, alpha.ctypes.data) == sbm.ERR_INVALID_ARG
    assert L.sherry_pack(W.ctypes.data, 0, 32, codes.ctypes.data, alpha.ctypes.data) == sbm.ERR_INVALID_ARG
    assert L.sherry_pack(W.ctypes.data, 4, 20, codes.ctypes.data, alpha.ctypes.data) == sbm.ERR_UNSUPPORTED_SHAPE
    W[2, 7] = np.inf
    assert L.sherry_pack(W.ctypes.data, 4, 32, codes.ctypes.data, alpha.ctypes.data) == sbm.ERR_NONFINITE
    with pytest.raises(sbm.SherryError):
        sbm.pack(W)
    # device entry points reject bad arguments before touching the GPU
    assert L.sherry_gemm(None, None, None, None, None, 1, 1, 32, None) == sbm.ERR_INVALID_ARG
    assert L.sherry_quant_act(None, 1, 32, None, None, None) == sbm.ERR_INVALID_ARG
    assert L.sherry_repack(None, 1, 32, None, None) == sbm.ERR_INVALID_ARG
    fake = ctypes.c_void_p(1 << 20)
    assert L.sherry_gemm(fake, fake, fake, fake, fake, 1, 1, 33, None) == sbm.ERR_UNSUPPORTED_SHAPE
    assert L.sherry_gemm(fake, fake, fake, fake, fake, 0, 1, 32, None) == sbm.ERR_INVALID_ARG
    assert L.sherry_gemm(ctypes.c_void_p((1 << 20) + 4), fake, fake, fake, fake, 1, 1, 32, None) == \
        sbm.ERR_INVALID_ARG                        # x_i8 not 16-byte aligned
    assert L.sherry_quant_act(fake, 1, 48, fake, fake, None) == sbm.ERR_UNSUPPORTED_SHAPE


def test_pack_thread_count_independent(lib):
    """alpha and codes do not depend on the number of host threads."""
    import subprocess, sys, json
    code = ("import numpy as np, sparse_bit_matmul_b200 as s, synth;"
            "W=synth.config_weights(1,0,4096,256); c,a=s.pack(W);"
            "print(int(c.astype(np.uint64).sum()), a.view(np.uint32).tolist()[:8])")
    outs = []
    for nt in ("1", "5"):
        env = dict(os.environ, OMP_NUM_THREADS=nt)
        outs.append(subprocess.check_output([sys.executable, "-c", code], env=env, cwd=ROOT).strip())
    assert outs[0] == outs[1]


def _function_spans(text):
    """(name, start, end) of every function body in a C/C++/CUDA source:
    the identifier before the parameter list of each '{' that opens a
    function, matched to its closing brace."""
    spans = []
    for m in re.finditer(r"\b([A-Za-z_]\w*)\s*\(([^;{}()]|\([^;{}()]*\))*\)\s*(const\s*)?\{", text):
        name = m.group(1)
        if name in ("if", "for", "while", "switch", "catch", "sizeof", "return"):
            continue
        depth, i = 0, m.end() - 1
        while i < len(text):
            if text[i] == "{":
                depth += 1
            elif text[i] == "}":
                depth -= 1
                if depth == 0:
                    break
            i += 1
        spans.append((name, m.start(), i))
    return spans


def test_async_entry_points_never_allocate_or_synchronise():
    """Allocation, freeing and host synchronisation appear in the device
    source only inside the host-synchronous entry points (sherry_reserve and
    its buffer growth, the status read with its reset); the per-call
    scratch clearing of sherry_gemm_noalloc is the only stream-ordered
    memset.  So none of the asynchronous entry points can reach them."""
    path = os.path.join(ROOT, "sparse_bit_matmul_b200", "csrc", "sherry_cuda.cu")
    text = open(path).read()
    text = re.sub(r"//[^\n]*", "", re.sub(r"/\*.*?\*/", "", text, flags=re.S))
    spans = _function_spans(text)
    allowed = {
        "cudaMalloc": {"grow_buffer"},
        "cudaFree": {"grow_buffer"},
        "cudaDeviceSynchronize": {"grow_buffer", "sherry_last_device_status"},
        "cudaStreamSynchronize": set(),
        "cudaMemset": {"grow_buffer", "sherry_last_device_status"},
        "cudaMemsetAsync": {"launch_tc_noalloc"},
        "cudaMallocAsync": set(),
        "cudaMallocManaged": set(),
    }
    callers = {"grow_buffer": {"sherry_reserve"}}
    for call, ok in allowed.items():
        for m in re.finditer(r"\b" + call + r"\s*\(", text):
            inner = [sp for sp in spans if sp[1] <= m.start() <= sp[2]]
            assert inner, f"{call} outside any function"
            name = min(inner, key=lambda sp: sp[2] - sp[1])[0]
            assert name in ok, f"{call} called in {name}"
    # grow_buffer itself is reached only from sherry_reserve
    for m in re.finditer(r"\bgrow_buffer\s*\(", text):
        inner = [sp for sp in spans if sp[1] <= m.start() <= sp[2] and sp[0] != "grow_buffer"]
        if not inner:
            continue                                   # its own definition
        name = min(inner, key=lambda sp: sp[2] - sp[1])[0]
        assert name in callers["grow_buffer"], f"grow_buffer called in {name}"
