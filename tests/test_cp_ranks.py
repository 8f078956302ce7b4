"""The context-parallel step's exchange order on CPU (gloo, world size 2):
run_step calls the four phases and the three all-gathers in the same order on
every rank, and each phase receives the ranks' buffers stacked in rank order.
The phases here are stand-ins that record what they receive (the real ones
launch the library's kernels, which need a GPU)."""
from __future__ import annotations

import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _FakeRank:
    def __init__(self, rank, torch):
        self.r, self.torch, self.seen = rank, torch, []

    def phase_a(self):
        t = self.torch
        return [t.full((2, 3), float(self.r)), t.full((2, 3), 10 + self.r, dtype=t.int32)]

    def phase_b(self, g_score, g_id):
        self.seen.append(("b", g_score.tolist(), g_id.tolist()))
        return [self.torch.full((4,), 100.0 + self.r)]

    def phase_c(self, g_p, swa_of=None, softmax_scale=0.0):
        self.seen.append(("c", g_p.tolist()))
        t = self.torch
        return [t.full((1, 2), 5.0 + self.r), t.full((1,), -1.0 - self.r)]

    def phase_d(self, g_o, g_lse):
        self.seen.append(("d", g_o.tolist(), g_lse.tolist()))


def _worker(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import torch
    import torch.distributed as dist

    from csa2_fp4_sparse_b200 import cp

    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        fr = _FakeRank(rank, torch)
        cp.run_step(fr, cp.torch_all_gather())
        q.put((rank, fr.seen))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_cp_exchange_order_gloo_world2():
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
    res = dict(q.get(timeout=10) for _ in range(2))
    for rank in (0, 1):
        seen = res[rank]
        assert [s[0] for s in seen] == ["b", "c", "d"]
        # phase B got both ranks' candidate lists, rank-major
        assert seen[0][1] == [[[0.0] * 3] * 2, [[1.0] * 3] * 2]
        assert seen[0][2] == [[[10] * 3] * 2, [[11] * 3] * 2]
        assert seen[1][1] == [[100.0] * 4, [101.0] * 4]
        assert seen[2][1] == [[[5.0, 5.0]], [[6.0, 6.0]]]
        assert seen[2][2] == [[-1.0], [-2.0]]
