"""Multi-process host logic of the benchmark on CPU (gloo, world size 2).

The attention path shards into independent replicas (no data-path
collective); what the N-GPU run adds is the timing aggregation -- time = max
over ranks, work = sum over ranks -- and the rank-0-only reporting, checked
here with two gloo ranks that report different times and work.
"""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms, work = bench.aggregate_ranks(torch, dist, "cpu", 10.0 + 5.0 * rank, 1000.0 * (rank + 1))
        q.put((rank, ms, work))
    finally:
        dist.destroy_process_group()


def test_aggregate_ranks_gloo_world2():
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
    for rank, ms, work in res:
        assert ms == 15.0      # max over ranks
        assert work == 3000.0  # sum over ranks


def test_aggregate_single_process_passthrough():
    import torch

    sys.path.insert(0, ROOT)
    import bench

    assert bench.aggregate_ranks(torch, None, "cpu", 3.5, 7.0) == (3.5, 7.0)


def test_visible_pair_counts():
    sys.path.insert(0, ROOT)
    import bench

    # brute-force count for small cases
    for lens, w in (([5], 0), ([5], 2), ([7, 3, 1], 3), ([128], 128), ([300], 128)):
        brute = sum(1 for n in lens for i in range(n) for j in range(i + 1) if w == 0 or i - j < w)
        assert bench.visible_pairs(lens, w) == brute
    # the bench workloads
    assert bench.visible_pairs([4096] * 4, 128) * 64 == 132_136_960
    assert bench.visible_pairs([8192] * 2, 0) * 64 == 4_295_491_584


@pytest.mark.parametrize("steps", [2])
def test_reference_arm_runs_on_cpu(steps, capsys):
    sys.path.insert(0, ROOT)
    import bench

    class A:
        pass

    a = A()
    a.steps, a.warmup, a.gpus = steps, 0, 1
    line = bench.run_reference(a)
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
