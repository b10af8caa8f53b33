"""The multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

Rows are independent, so ranks shard the batch (each draws its own seeded
rows) and only the per-run timing vector crosses ranks (an all-reduce MAX).
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times = [0.1 * (rank + 1), 0.5 - 0.1 * rank, 1.0]
        mx = bench.max_over_ranks(times, world, torch.device("cpu"))
        seeds = [bench.rank_seed(7, rank)]
        gathered = [None] * world
        dist.all_gather_object(gathered, seeds)
        bench.barrier(world)
        out.put((rank, mx, gathered))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_max_and_draw_distinct_rows():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, gathered in res:
        assert mx == pytest.approx([0.2, 0.5, 1.0])
        assert gathered[0] != gathered[1]  # each rank draws its own rows


def test_reference_arm_other_ranks_do_nothing(monkeypatch):
    import bench

    args = type("A", (), {"workload": "sweep-quick", "steps": 1, "warmup": 3, "ref_rows": 1})()
    assert bench.reference_arm(args, rank=1, world=2) is None


def test_single_rank_max_is_identity():
    import bench

    assert bench.max_over_ranks([1.0, 2.0], 1, torch.device("cpu")) == [1.0, 2.0]
