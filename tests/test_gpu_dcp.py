"""Context-parallel indexer ([post, "NVFP4 indexer DCP"]) on one GPU.

The ranks of a context-parallel group are emulated as consecutive launches of
msa_indexer_score_part on one GPU (they do not wait on one another).  Each
part must write exactly its blocks, with the values the full launch writes
for them (bit for bit), and the element-wise max of the parts must give the
full launch's block scores and selection.  The merged parts and the
selection made from them are also compared with the float64 oracle, and the
product orchestration (dcp.select) runs once with a single rank.  The exchange
between ranks is covered on CPU (tests/test_dcp_cpu.py).
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_decode_b200 as msa
from block_sparse_attention_decode_b200 import build as msa_build
from block_sparse_attention_decode_b200 import dcp, synth
import oracle
from tests import parity

pytestmark = pytest.mark.gpu

CASES = [
    ("ragged_t1", dict(batch=4, seq_lens=[5000, 300, 2049, 1], q_tokens=1, paged=True, seed=92), (2, 3, 4)),
    ("t8", dict(batch=2, seq_lens=[9000, 3000], q_tokens=8, paged=True, seed=93), (2, 4, 7)),
    ("t8_exact", dict(batch=2, seq_lens=[9000, 2100], q_tokens=8, paged=True, seed=94,
                      idx_exact=True), (3,)),
    ("fp8idx", dict(batch=2, seq_lens=[6000, 700], q_tokens=2, paged=False, seed=95,
                    idx_fp8=True), (4,)),
]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    msa_build.build()
    msa.load()


def _scores(w, part=None, nparts=None, fill=float("nan")):
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    ts = torch.full((w.batch, w.q_tokens, 4, w.max_pages * 128), fill, device="cuda")
    bs = torch.full((w.batch, w.q_tokens, 4, w.max_pages), fill, device="cuda")
    if part is None:
        msa.msa_indexer_score(cache, seqs, w.qi, w.s_qi, ts, bs, ws)
    else:
        msa.msa_indexer_score_part(cache, seqs, w.qi, w.s_qi, ts, bs, part, nparts, ws)
    torch.cuda.synchronize()
    assert msa.msa_get_last_error(ws)[0] == msa.MSA_OK
    assert ws[64:72].view(torch.int32).tolist() == [0, 0]     # work counters reset
    return ts.cpu().numpy(), bs.cpu().numpy()


def _select(w, bs):
    seqs = msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    sel = torch.empty(w.batch, w.q_tokens, 4, 16, dtype=torch.int32, device="cuda")
    msa.msa_block_maxpool_topk(torch.from_numpy(bs).cuda(), False, seqs, sel, ws)
    torch.cuda.synchronize()
    return sel.cpu().numpy()


@pytest.mark.parametrize("name,kw,nparts_list", CASES, ids=[c[0] for c in CASES])
def test_parts_write_their_blocks_bit_exactly(name, kw, nparts_list):
    w = synth.make_workload(name, device="cuda", **kw)
    ts_full, bs_full = _scores(w)
    lens = w.seq_lens.cpu().tolist()
    for nparts in nparts_list:
        merged = np.full_like(bs_full, -np.inf)
        for part in range(nparts):
            ts, bs = _scores(w, part, nparts)
            for b, L in enumerate(lens):
                nblk = (L + 127) // 128
                lo, hi = dcp.block_range(nblk, part, nparts)
                # this part's blocks: the full launch's values, bit for bit
                assert np.array_equal(bs[b, :, :, lo:hi], bs_full[b, :, :, lo:hi]), (name, nparts, part, b)
                assert np.array_equal(ts[b, :, :, lo * 128:hi * 128], ts_full[b, :, :, lo * 128:hi * 128])
                # nothing else written
                assert np.isnan(bs[b, :, :, :lo]).all() and np.isnan(bs[b, :, :, hi:]).all()
                assert np.isnan(ts[b, :, :, :lo * 128]).all() and np.isnan(ts[b, :, :, hi * 128:]).all()
            _, bs_inf = _scores(w, part, nparts, fill=float("-inf"))
            merged = np.maximum(merged, bs_inf)
        for b, L in enumerate(lens):
            nblk = (L + 127) // 128
            assert np.array_equal(merged[b, :, :, :nblk], bs_full[b, :, :, :nblk]), (name, nparts, b)
        assert np.array_equal(_select(w, merged), _select(w, bs_full)), (name, nparts)


def test_part_arguments_checked():
    w = synth.make_workload("dcp_args", 1, [500], 1, paged=False, seed=96, device="cuda")
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    bs = torch.empty(1, 1, 4, w.max_pages, device="cuda")
    for part, nparts in ((0, 0), (2, 2), (-1, 2), (0, msa.MAX_PARTS + 1)):
        with pytest.raises(msa.MsaError) as e:
            msa.msa_indexer_score_part(cache, seqs, w.qi, w.s_qi, None, bs, part, nparts, ws)
        assert e.value.status == msa.MSA_ERR_INVALID_ARG


# ------------------------------------------------------ against the oracle --
# The parts' merged block scores and the selection made from them, compared
# with the float64 oracle (not with the GPU's own full launch), at the stated
# tolerances: scores 1e-3 relative, selection exact up to near-ties
# ([post, "NVFP4 indexer DCP"]: the selection stays exact).
ORACLE_CASES = [
    ("ragged_t1", dict(batch=4, seq_lens=[5000, 300, 2049, 7000], q_tokens=1, paged=True, seed=97), (2, 3, 4)),
    ("t8", dict(batch=2, seq_lens=[9000, 3000], q_tokens=8, paged=True, seed=98), (2, 3, 4)),
]


def _oracle_block_scores(w):
    c, _ = parity.host_cache(w)
    rows = oracle.all_rows(c)
    _, rbs = oracle.indexer(c, w.qi.cpu().numpy(), w.s_qi, rows, token_scores=False)
    return c, rows, rbs


@pytest.mark.parametrize("name,kw,nparts_list", ORACLE_CASES, ids=[c[0] for c in ORACLE_CASES])
def test_merged_parts_match_the_oracle(name, kw, nparts_list):
    w = synth.make_workload(name + "_orc", device="cuda", **kw)
    c, rows, rbs = _oracle_block_scores(w)
    ref_sel = oracle.select(c, rows, rbs)
    nvis = np.array([(int(c.seq_lens[b]) - c.q_tokens + t) // 128 + 1 for b, t in rows])
    for nparts in nparts_list:
        merged = None
        for part in range(nparts):
            _, bs = _scores(w, part, nparts, fill=float("-inf"))
            part_t = torch.from_numpy(bs)
            # the element-wise max the all-reduce of dcp.merge_block_scores performs
            merged = part_t if merged is None else torch.maximum(merged, part_t)
        g = merged.numpy().reshape(len(rows), 4, -1)
        for r, (b, t) in enumerate(rows):
            nblk = (int(c.seq_lens[b]) + 127) // 128
            parity.check_scores(g[r, :, :nblk], rbs[r, :, :nblk], "%s nparts %d row %d" % (name, nparts, r))
        gsel = _select(w, merged.numpy()).reshape(len(rows), 4, 16)
        parity.check_selection(gsel, ref_sel, rbs, nvis, "%s nparts %d" % (name, nparts))


def test_dcp_select_world_one_matches_the_oracle():
    """The product orchestration (dcp.select: part launch, merge, top-16) run
    by a single process with no process group (one rank, one part)."""
    w = synth.make_workload("dcp_select", 3, [6000, 2049, 400], 8, paged=True, seed=99, device="cuda")
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    bs = torch.empty(w.batch, w.q_tokens, 4, w.max_pages, device="cuda")
    sel = torch.empty(w.batch, w.q_tokens, 4, 16, dtype=torch.int32, device="cuda")
    dcp.select(cache, seqs, w.qi, w.s_qi, bs, sel, ws)
    torch.cuda.synchronize()
    assert msa.msa_get_last_error(ws)[0] == msa.MSA_OK
    c, rows, rbs = _oracle_block_scores(w)
    g = bs.cpu().numpy().reshape(len(rows), 4, -1)
    for r, (b, t) in enumerate(rows):
        nblk = (int(c.seq_lens[b]) + 127) // 128
        parity.check_scores(g[r, :, :nblk], rbs[r, :, :nblk], "dcp.select row %d" % r)
    nvis = np.array([(int(c.seq_lens[b]) - c.q_tokens + t) // 128 + 1 for b, t in rows])
    parity.check_selection(sel.cpu().numpy().reshape(len(rows), 4, 16), oracle.select(c, rows, rbs),
                           rbs, nvis, "dcp.select")
