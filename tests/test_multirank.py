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


def test_head_range_partitions_the_heads():
    from sparse_attention_video_head_b200.shard import head_range
    for H in (1, 7, 24, 40):
        for world in (1, 2, 3, 8):
            blocks = [head_range(H, world, r) for r in range(world)]
            assert blocks[0][0] == 0 and blocks[-1][1] == H
            assert all(blocks[r][1] == blocks[r + 1][0] for r in range(world - 1))
            sizes = [b - a for a, b in blocks]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    with pytest.raises(ValueError):
        head_range(4, 2, 2)


def _shard_rank(rank, world, port, q):
    """One rank of a head-sharded layer on CPU: the oracle plays the per-head computation, the
    ranks' output blocks are gathered over gloo and compared with the unsharded layer."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import bench
    from oracle import oracle as O
    from sparse_attention_video_head_b200 import inputs as I
    from sparse_attention_video_head_b200.shard import head_range
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = I.CONFIGS["tiny"]
        import dataclasses
        cfg = dataclasses.replace(cfg, H=3)  # 3 heads over 2 ranks: blocks of 2 and 1
        h0, h1 = head_range(cfg.H, world, rank)
        data = bench.gen_inputs(cfg, heads=range(h0, h1))
        outs = []
        for i in range(h1 - h0):
            res = O.layer_head(data["q"][0, i], data["k"][0, i], data["v"][0, i], cfg.nQ, cfg.nK, cfg.iters, 0.9,
                               float(np.float32(cfg.scale)), uq=data["uq"][0, i], uk=data["uk"][0, i])
            outs.append(res["o"])
        local = torch.from_numpy(np.stack(outs))
        pad = torch.zeros((head_range(cfg.H, world, 0)[1],) + tuple(local.shape[1:]), dtype=local.dtype)
        pad[: local.shape[0]] = local
        got = [torch.zeros_like(pad) for _ in range(world)]
        dist.all_gather(got, pad)
        if rank == 0:
            full = torch.cat([g[: b - a] for g, (a, b) in zip(got, [head_range(cfg.H, world, r) for r in range(world)])])
            ref_data = bench.gen_inputs(cfg)
            ref = np.stack([O.layer_head(ref_data["q"][0, h], ref_data["k"][0, h], ref_data["v"][0, h], cfg.nQ, cfg.nK,
                                         cfg.iters, 0.9, float(np.float32(cfg.scale)), uq=ref_data["uq"][0, h],
                                         uk=ref_data["uk"][0, h])["o"] for h in range(cfg.H)])
            q.put(float(np.abs(full.numpy() - ref).max()))
        slowest = bench.max_over_ranks([10.0, 12.0][rank], world, dist, "cpu")
        q.put(("ms", rank, bench.whole_job_ms_per_layer(slowest, world, sharded=True)))
    finally:
        dist.destroy_process_group()


def test_head_sharded_layer_equals_the_unsharded_one_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    items = [q.get(timeout=10) for _ in range(3)]
    diffs = [x for x in items if not isinstance(x, tuple)]
    assert diffs == [0.0]  # the same per-head inputs and arithmetic, whichever rank computes a head
    assert sorted(x[2] for x in items if isinstance(x, tuple)) == [12.0, 12.0]  # one layer per step
