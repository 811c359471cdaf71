"""Host-side logic of the multi-GPU benchmark, run as two gloo ranks on the CPU: every
rank owns a disjoint batch element of the workload (no data-path collective), the union
covers the global batch, and the reported time is the maximum over ranks."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = bench.rank_heads(1, 32, rank)
        t = bench.max_over_ranks(1.0 + rank, world)  # each rank's own "time"
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        out[rank] = (t, gathered)
    finally:
        dist.destroy_process_group()


def test_two_ranks_partition_heads_and_take_max():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    for rank in range(world):
        t, gathered = res[rank]
        assert t == 2.0  # max over ranks
        flat = [p for g in gathered for p in g]
        assert len(flat) == len(set(flat)) == world * 32
        assert {b for b, _ in flat} == {0, 1}
