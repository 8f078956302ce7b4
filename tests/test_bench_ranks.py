"""The benchmark's multi-process path on CPU (gloo, world size 2): the host-side
reductions (max over ranks of the time, sum over ranks of the query tokens),
the whole-job rate, and the reference arm launched under torchrun, where rank
0 alone prints the JSON line and the other rank exits 0 without work."""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench

    r = bench.Ranks(device="cpu", timeout_s=60)
    try:
        t_ms = 100.0 + 50.0 * rank          # rank 1 is the slow one
        tokens = 3 + 2 * rank               # ranks decode different batches
        mx = r.allmax(t_ms)
        tot = r.allsum(tokens)
        r.barrier()
        q.put((rank, mx, tot, bench.whole_job_rate(tot, 4, 4 * mx)))
    finally:
        r.close()


def test_ranks_reductions_gloo_world2():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, tot, rate in res:
        assert mx == 150.0           # max over ranks
        assert tot == 8.0            # 3 + 5 tokens
        assert abs(rate - 8 / 0.150) < 1e-9  # all tokens over the slowest rank's time per step


def test_whole_job_rate_single():
    import bench

    assert bench.whole_job_rate(4, 10, 2000.0) == 20.0


def test_reference_arm_under_torchrun_world2():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--config", "1",
           "--cpu-seconds", "0.5"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1  # rank 0 only
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "qtok/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["unit"] == d["unit"]


def test_source_digest_ignores_comments_only():
    import bench

    a = "int f(int x) {\n  return x + 1;  // one\n}\n/* block\n comment */\n"
    b = "// header\nint f(int x) {   return x + 1; }\n"
    c = "int f(int x) {\n  return x + 2;\n}\n"
    assert bench.source_digest(a) == bench.source_digest(b)
    assert bench.source_digest(a) != bench.source_digest(c)


def test_algorithmic_flops_closed_form():
    import bench
    from synth.workloads import CONFIGS, make_workload

    w = make_workload(CONFIGS[4])
    f = bench.algorithmic_flops(w)
    c = w.cfg
    n_pos = 4 * 1048576  # one query token per sequence, every position visible
    assert f["scan"] == n_pos * c.H_I * c.d_I * 2
    assert f["rescore"] == 4 * c.P * 8 * 4 * c.H_I * c.d_I * 2  # 4 selectors, full pools
    assert f["attend"] == 4 * c.K * 20 * c.Hq * c.D * 4
