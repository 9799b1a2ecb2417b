"""Indexer context parallelism across GPUs ([post, "NVFP4 indexer DCP"]).

Without it, every GPU of a tensor-parallel group scores its own index head
over the whole context, so each indexer layer reads the index cache once per
GPU.  With it, each rank scores all four index heads over its own part of
every sequence's pages (``msa_indexer_score_part``), the parts' block scores
are combined by one element-wise max all-reduce (NCCL over NVLink between
GPUs), and the top-16 is then taken from the full block scores, so the
selection is exactly the single-GPU one.  Each rank reads only the pages of
its part: its page table may leave the other parts' entries unset.

What the all-reduce carries per step is 4 bytes per (sequence, token, group,
block) -- 128 KB per 128K-token sequence at 8 query tokens -- against 9.4 MB
of index keys per such sequence, of which each rank now reads only its part.

Host orchestration only; the scoring and the selection run in libmsa's
kernels, the exchange in the process group's collective.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import Cache, Seqs, msa_block_maxpool_topk, msa_indexer_score_part


def block_range(nblk: int, part: int, nparts: int) -> tuple[int, int]:
    """Logical blocks [lo, hi) of a sequence of nblk blocks that part `part`
    of `nparts` scores (the rule msa_indexer_score_part applies)."""
    return nblk * part // nparts, nblk * (part + 1) // nparts


def _rank_world(group):
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(group), dist.get_world_size(group)
    return 0, 1


def merge_block_scores(block_scores: torch.Tensor, group=None) -> torch.Tensor:
    """In place: the element-wise max over the ranks of `group`.  Each rank's
    tensor holds its part's block scores and -inf elsewhere."""
    _, world = _rank_world(group)
    if world > 1:
        dist.all_reduce(block_scores, op=dist.ReduceOp.MAX, group=group)
    return block_scores


def indexer_scores(cache: Cache, seqs: Seqs, qi, s_qi: float, block_scores: torch.Tensor, ws,
                   group=None, stream=None) -> torch.Tensor:
    """Block scores [B][T][4][max_pages] of the whole context on every rank:
    this rank's part scored here, the rest received from the other ranks."""
    rank, world = _rank_world(group)
    stream = stream or torch.cuda.current_stream()
    with torch.cuda.stream(stream):
        block_scores.fill_(float("-inf"))
        msa_indexer_score_part(cache, seqs, qi, s_qi, None, block_scores, rank, world, ws, stream)
        return merge_block_scores(block_scores, group)


def select(cache: Cache, seqs: Seqs, qi, s_qi: float, block_scores: torch.Tensor, sel, ws,
           group=None, stream=None):
    """The selection [B][T][4][16] from the context-parallel index scores."""
    stream = stream or torch.cuda.current_stream()
    indexer_scores(cache, seqs, qi, s_qi, block_scores, ws, group, stream)
    msa_block_maxpool_topk(block_scores, False, seqs, sel, ws, stream)
    return sel
