"""The N > 1 path of bench.py on CPU with gloo, world size 2: every rank runs its own layer
(replicas; the layer's heads are independent, so nothing is exchanged on the data path), the step
time is the max over ranks, and the whole-job value is per layer."""
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


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [120.0, 135.5][rank]  # a slower rank 1
        slowest = bench.max_over_ranks(local_ms, world, dist, "cpu")
        q.put((rank, slowest, bench.whole_job_ms_per_layer(slowest, world)))
    finally:
        dist.destroy_process_group()


def test_step_time_is_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[1] for g in got] == [135.5, 135.5]
    assert [g[2] for g in got] == [135.5 / 2, 135.5 / 2]


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.0, 1, None, "cpu") == 7.0
    assert bench.whole_job_ms_per_layer(7.0, 1) == 7.0
