"""Context-parallel indexer ([post, "NVFP4 indexer DCP"]): host logic on CPU.

The split of every sequence's blocks into parts, and the exchange that
combines the parts' block scores (an element-wise max all-reduce), run here
with two gloo ranks.  Each rank's partial block scores come from the oracle
restricted to its part (what msa_indexer_score_part writes on the GPU; that
kernel's part output is checked against the full launch in
tests/test_gpu_dcp.py); after the exchange both ranks must hold the oracle's
full block scores and make the oracle's full selection.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from block_sparse_attention_decode_b200 import dcp, synth
from tests import parity


def test_parts_tile_every_sequence():
    for nblk in list(range(0, 40)) + [1023, 1024, 2048]:
        for nparts in range(1, 9):
            spans = [dcp.block_range(nblk, p, nparts) for p in range(nparts)]
            assert spans[0][0] == 0 and spans[-1][1] == nblk
            assert all(spans[i][1] == spans[i + 1][0] for i in range(nparts - 1))
            sizes = [hi - lo for lo, hi in spans]
            assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # the same batch on both ranks (context parallelism splits one batch)
        w = synth.make_workload("dcp", 3, [5000, 300, 2049], 4, paged=True, seed=91)
        c, _ = parity.host_cache(w)
        rows = oracle.all_rows(c)
        _, full = oracle.indexer(c, w.qi.numpy(), w.s_qi, rows, token_scores=False)
        full32 = full.astype(np.float32)
        part = np.full_like(full32, -np.inf)
        for r, (b, t) in enumerate(rows):
            nblk = (int(c.seq_lens[b]) + 127) // 128
            lo, hi = dcp.block_range(nblk, rank, world)
            part[r, :, lo:hi] = full32[r, :, lo:hi]
        merged = dcp.merge_block_scores(torch.from_numpy(part).clone()).numpy()
        nblks = [(int(c.seq_lens[b]) + 127) // 128 for b, _ in rows]
        same = all(np.array_equal(merged[r, :, :n], full32[r, :, :n]) for r, n in enumerate(nblks))
        sel_merged = oracle.select(c, rows, merged.astype(np.float64))
        sel_full = oracle.select(c, rows, full32.astype(np.float64))
        q.put((rank, same, bool(np.array_equal(sel_merged, sel_full)),
               bool(np.array_equal(part, full32))))
    finally:
        dist.destroy_process_group()


def test_two_ranks_merge_to_the_full_selection():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, same, sel_same, part_was_full in res:
        assert same and sel_same, rank
        assert not part_was_full, rank          # each rank really held only a part


def test_single_process_merge_is_identity():
    x = torch.randn(2, 3, 4, 5)
    assert torch.equal(dcp.merge_block_scores(x.clone()), x)
