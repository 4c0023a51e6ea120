"""The multi-GPU benchmark path runs independent replicas (no data-path
collective); its host logic is checked here with two gloo ranks on the CPU:
disjoint batch pools, the max-over-ranks time, and the whole-job rate."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ids = bench.rank_batch_ids(rank)
        gathered = [None] * world
        dist.all_gather_object(gathered, ids)
        elapsed = 10.0 + 5.0 * rank           # the slower rank decides
        m = bench.max_over_ranks(elapsed, world, "cpu")
        rate = bench.aggregate_rate(65536 * 20, world, m)
        out[rank] = (gathered, m, rate)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        gathered, m, rate = out[r]
        assert set(gathered[0]).isdisjoint(gathered[1]), "ranks must draw different batches"
        assert m == 15.0
        assert abs(rate - 65536 * 20 * 2 / 0.015) < 1e-6
    assert bench.max_over_ranks(3.0, 1) == 3.0
