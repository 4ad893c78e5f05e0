"""Host logic of bench.py on CPU: byte accounting, max-over-ranks timing and
the reference arm under a 2-rank gloo launch (no GPU)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_algorithmic_bytes():
    # 5-bit codes (1.25 bit/weight) + fp32 alpha + int8 x + fp32 scale
    assert bench.algorithmic_bytes(1, 4096, 4096) == 4096 * 4096 * 5 // 32 + 4 * 4096 + 4096 + 4
    codes = sum(N * K * 5 // 32 for K, N in bench.PROJ_SHAPES)
    assert codes * 32 == 671_088_640                     # 32 layer copies: 671 MB > 126 MB L2
    total = sum(bench.algorithmic_bytes(1, K, N) for K, N in bench.PROJ_SHAPES)
    assert total == codes + 4 * (4096 + 14336 + 4096) + (4096 + 4096 + 14336) + 3 * 4


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    w, r, _ = bench.dist_setup(world, need_cuda=False)
    v = bench.max_over_ranks(1.5 + r, w)
    bench.barrier(w)
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((r, w, v))


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, 2, 2.5), (1, 2, 2.5)]


def test_reference_arm_two_ranks_prints_one_line():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_cpu_lut_leg_reports_a_rate():
    r = bench.cpu_lut_baseline(0.2)
    assert "unavailable" not in r, r
    assert r["value"] > 0 and r["unit"] == "GB/s" and r["cores"] >= 1
    assert r["kind"].startswith("page_cpu_lut_")
