"""Multi-process host logic of the benchmark (world size 2, gloo, CPU): per-rank times are
combined as the max over ranks and token counts as the sum, and the JSON line's `value` is
whole-job throughput.  The decode path itself has no collective (independent replicas)."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime

    import bench

    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        my_ms = 10.0 * (rank + 1)           # rank 1 is slower
        mx = bench.aggregate(my_ms, "max", world)
        tot = bench.aggregate(100.0, "sum", world)
        q.put((rank, mx, tot, bench.dist_env()))
    finally:
        dist.destroy_process_group()


def test_rank_aggregation_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, tot, env in res:
        assert mx == 20.0            # max over ranks
        assert tot == 200.0          # sum over ranks
        assert env == (2, rank, rank)


def test_phase_summary_and_aggregate_single_rank():
    import numpy as np

    sys.path.insert(0, ROOT)
    import bench

    assert bench.aggregate(3.5, "max", 1) == 3.5
    # P = 4 CTAs in k = 2 slot groups; stamp j of CTA c at layer l: 10 us * l + 0.1 us * j + c ns
    L, P = 3, 4
    tr = np.zeros((L, P, 24), np.int64)
    for l in range(L):
        for c in range(P):
            tr[l, c, :15] = 10000 * l + 100 * np.arange(15) + c
    s = bench.phase_summary(tr, k=2)
    assert s["layer_total"] == 10.0
    assert abs(s["x_wait"] - 0.1) < 1e-9
    assert abs(s["combine"] - 0.1) < 1e-9
    # logits, all CTAs: first receipt (CTA 0, stamp 4) - last publish (CTA 3, stamp 2) = 200 - 3 ns
    assert abs(s["exchange_latency"]["logits"] - 0.197) < 1e-9
    # h inside a slot group {0, 1} / {2, 3}: 100 ns - 1 ns
    assert abs(s["exchange_latency"]["h"] - 0.099) < 1e-9
    # y among the CTAs of one part (CTAs 0 and 2): 100 ns - 2 ns
    assert abs(s["exchange_latency"]["y"] - 0.098) < 1e-9
    # x from layer l's last publish (stamp 14) to layer l + 1's first receipt (stamp 1): 10 us
    # + 100 ns - 1,400 ns - 1 ns
    assert abs(s["exchange_latency"]["x"] - 8.699) < 1e-9
