"""Multi-process (world size 2, gloo, CPU) checks of the benchmark's rank logic.

The decode path shards by sequence, so ranks share nothing on the data path:
each rank builds its own batch (its own seed) and the only collectives are the
timing barrier and the max over ranks of the measured time.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from block_sparse_attention_decode_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, w, lr = bench.rank_info()
        assert (r, w, lr) == (rank, world, rank)
        # each rank decodes its own batch: same shapes, different bytes
        kw = dict(synth.WORKLOADS["ctx4k_b1_t1"])
        kw["seed"] += bench.rank_seed_offset(rank)
        wl = synth.make_workload("dist", **kw)
        digest = int(wl.k_data.to(torch.int64).sum().item())
        bench.barrier(world)
        # max over ranks of a per-rank time
        t_max = bench.max_over_ranks(1.5 + rank, world)
        gathered = [None] * world
        dist.all_gather_object(gathered, digest)
        q.put((rank, t_max, gathered))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_by_seed_and_take_max_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert all(t == 2.5 for _, t, _ in res)                 # max over ranks, on every rank
    digests = res[0][2]
    assert digests == res[1][2] and digests[0] != digests[1]   # different data per rank


def test_single_rank_helpers_without_process_group():
    assert bench.max_over_ranks(3.25, 1) == 3.25
    bench.barrier(1)
    assert bench.rank_seed_offset(0) == 0 and bench.rank_seed_offset(3) != 0
