"""Host logic of the multi-GPU benchmark path, on CPU with the gloo backend
(world size 2): each rank runs an independent workload (weak scaling, no
collective on the data path), and the reported time is the maximum over
ranks, taken by one all-reduce at the same point on every rank."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = 10.0 + 5.0 * rank                     # rank 1 is the slow one
        ms_max = bench.max_over_ranks(dist, world, my_ms, device="cpu")
        value = bench.weak_scaling_value(world, 1000, ms_max)
        seed = bench.rank_seed(30, rank)
        # the reference arm does no work on ranks other than 0
        if rank != 0:
            bench.run_reference(type("A", (), {"workload": "tiny_f32", "steps": 1, "warmup": 0})())
        out.put((rank, ms_max, value, seed))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_sharding():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    assert [r[1] for r in res] == [15.0, 15.0]                 # max over ranks, seen by every rank
    assert res[0][2] == pytest.approx(2 * 1000 / 15e-3)        # units of all ranks / slowest time
    assert res[0][3] != res[1][3]                              # independent inputs per rank


def test_single_rank_is_identity():
    assert bench.max_over_ranks(None, 1, 3.5) == 3.5
    assert bench.weak_scaling_value(1, 50, 2.0) == pytest.approx(25000.0)
