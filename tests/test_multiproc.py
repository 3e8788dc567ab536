"""The benchmark's multi-rank path on CPU: two gloo ranks.

Each rank decodes its own batch of the workload (weak scaling, no data-path
collective); the only cross-rank traffic is the barrier and the max-over-ranks
of the measured times.  These tests exercise that bookkeeping without a GPU.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from synth import config_spec
        # rank r measured (10 + r) ms for 4 steps and (2 + r) ms of attention
        ms_step, attn_ms, value = bench.aggregate(dist, world, 4, 10.0 + rank, 2.0 + rank, 1_000_000)
        spec = config_spec("gqa70b", shard=rank)
        same = config_spec("mha7b", shard=rank)
        bench.barrier(dist)
        q.put((rank, ms_step, attn_ms, value, spec["lens"][:3], spec["seed"], same["lens"][:2]))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_and_shards():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms_step, attn_ms, value, lens, seed, mha in res:
        assert ms_step == pytest.approx(11.0 / 4)             # slowest rank's time
        assert attn_ms == pytest.approx(3.0)
        assert value == pytest.approx(world * 1_000_000 / (11.0 / 4 * 1e-3) / 1e9)
        assert mha == [4096, 4096]                             # uniform workload: same shape
    assert res[0][4] != res[1][4], "ranks must decode different batches"
    assert res[0][5] != res[1][5]
