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


def _forward_worker(rank, world, port, out):
    """Each rank draws its own heads as bench.py does and runs the forward on them (the
    oracle stands in for the device kernels here); the gathered outputs must be the global
    batch's forward."""
    import numpy as np

    import bench
    import oracle
    from linear_attention_linattn_b200 import inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, n, d = 1, 3, 70, 8
        q, k, v = inputs.forward_qkv(5, B * world, H, n, d, True,
                                     heads=bench.rank_heads(B, H, rank))
        mine = oracle.forward(q.reshape(B, H, n, d), k.reshape(B, H, n, d),
                              v.reshape(B, H, n, d), True)
        gathered = [None] * world
        dist.all_gather_object(gathered, np.asarray(mine))
        out[rank] = np.concatenate(gathered, axis=0)
    finally:
        dist.destroy_process_group()


def test_two_ranks_forward_their_heads_and_cover_the_global_batch():
    import numpy as np

    import oracle
    from linear_attention_linattn_b200 import inputs
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_forward_worker, args=(world, port, out), nprocs=world,
                           start_method="spawn")
        res = dict(out)
    q, k, v = inputs.forward_qkv(5, world, 3, 70, 8, True)
    ref = oracle.forward(q, k, v, True)
    for rank in range(world):
        assert res[rank].shape == ref.shape
        assert np.array_equal(res[rank], ref)
