"""GPU parity of the shared-prefix path ([post, "AMD GPU support", "NVFP4 MSA
kernel"]: a shared-prefix page is dequantised once for the requests that
share it): msa_indexer_score_grouped / msa_decode_grouped on caches whose
sequences share their first blocks' pages, against the float64 oracle (which
reads every sequence's pages through its page table) and against the
ungrouped calls on the same cache, which read each shared page once per
sequence."""
import zlib

import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_decode_b200 as msa
from block_sparse_attention_decode_b200 import build as msa_build
from block_sparse_attention_decode_b200 import synth
from tests import parity

pytestmark = pytest.mark.gpu

# (name, batch lengths, q_tokens, prefix groups [(users, shared blocks)], extra)
CASES = [
    ("t8_two_groups", [9000, 7000, 12000, 3000, 5000], 8, [(3, 40), (2, 10)], {}),
    ("t1_one_group", [20000, 16000, 18000, 30000], 1, [(4, 100)], {}),
    ("t1_mixed", [5000, 4000, 6000, 2100], 1, [(1, 0), (2, 25), (1, 0)], {}),
    ("t4_full_prefix", [4096 + 200, 4096 + 300, 4096 + 4], 4, [(3, 32)], {}),
    ("t8_fp8idx", [6000, 6500, 7000], 8, [(3, 30)], {"idx_fp8": True}),
    ("t8_exact", [6000, 6500, 7000], 8, [(3, 30)], {"idx_exact": True}),
]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    msa_build.build()
    msa.load()


def _workload(name, lens, T, groups, extra):
    return synth.make_workload(name, len(lens), lens, T, paged=True, seed=zlib.crc32(name.encode()) % 10000,
                               device="cuda", prefix_groups=groups, **extra)


def _scores(w, groups=None, token_level=False):
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    bs = torch.full((w.batch, w.q_tokens, 4, w.max_pages), float("nan"), device="cuda")
    ts = None
    if token_level:
        ts = torch.full((w.batch, w.q_tokens, 4, w.max_pages * 128), float("nan"), device="cuda")
    if groups is None:
        msa.msa_indexer_score(cache, seqs, w.qi, w.s_qi, ts, bs, ws)
    else:
        msa.msa_indexer_score_grouped(cache, seqs, groups, w.qi, w.s_qi, ts, bs, ws)
    torch.cuda.synchronize()
    st = msa.msa_get_last_error(ws)
    assert st[0] == msa.MSA_OK, st
    assert ws[64:72].view(torch.int32).tolist() == [0, 0]     # work counters reset
    return bs.cpu().numpy(), None if ts is None else ts.cpu().numpy()


def test_generator_shares_the_prefix_pages():
    w = _workload("gen", [3000, 2600, 4000], 1, [(3, 12)], {})
    pt = w.page_table.cpu().numpy()
    assert (pt[1, :12] == pt[0, :12]).all() and (pt[2, :12] == pt[0, :12]).all()
    nblk = [(L + 127) // 128 for L in (3000, 2600, 4000)]
    own = np.concatenate([pt[b, 12:nblk[b]] for b in range(3)])
    assert len(set(own.tolist()) | set(pt[0, :12].tolist())) == 12 + len(own)   # the rest is private
    assert w.num_pages == 12 + sum(n - 12 for n in nblk)


@pytest.mark.parametrize("name,lens,T,groups,extra", CASES, ids=[c[0] for c in CASES])
def test_grouped_indexer_matches_oracle_and_ungrouped(name, lens, T, groups, extra):
    w = _workload(name, lens, T, groups, extra)
    g = msa.PrefixGroups.of(groups)
    bs_g, ts_g = _scores(w, g, token_level=True)
    bs_u, ts_u = _scores(w, None, token_level=True)
    c, _ = parity.host_cache(w)
    rows = oracle.all_rows(c)
    rts, rbs = oracle.indexer(c, w.qi.cpu().numpy(), w.s_qi, rows, ctx_cap=w.max_pages * 128)
    gb = bs_g.reshape(len(rows), 4, -1)
    gt = ts_g.reshape(len(rows), 4, -1)
    for r, (b, t) in enumerate(rows):
        L = int(c.seq_lens[b])
        nblk = (L + 127) // 128
        pos = L - T + t
        parity.check_scores(gb[r, :, :nblk], rbs[r, :, :nblk], "%s block scores row %d" % (name, r))
        ref_t = np.full((4, nblk * 128), -np.inf)
        ref_t[:, :pos + 1] = rts[r, :, :pos + 1]
        parity.check_scores(gt[r, :, :nblk * 128], ref_t, "%s token scores row %d" % (name, r))
    # bit for bit the scores of the ungrouped indexer, which reads each
    # shared page once per sequence (the same products summed in the same
    # order; only the tile a query row sits in differs)
    for b in range(len(lens)):
        nblk = (lens[b] + 127) // 128
        assert np.array_equal(bs_g[b, :, :, :nblk], bs_u[b, :, :, :nblk]), (name, b)


@pytest.mark.parametrize("name,lens,T,groups,extra", CASES[:3], ids=[c[0] for c in CASES[:3]])
def test_grouped_decode_matches_oracle(name, lens, T, groups, extra):
    w = _workload(name, lens, T, groups, extra)
    g = msa.PrefixGroups.of(groups)
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    out = torch.empty(w.batch, T, 64, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(w.batch, T, 4, 16, dtype=torch.int32, device="cuda")
    msa.msa_decode_grouped(cache, seqs, g, w.qi, w.s_qi, w.q, w.s_q, w.softmax_scale, out, sel, ws)
    torch.cuda.synchronize()
    assert msa.msa_get_last_error(ws)[0] == msa.MSA_OK
    c, _ = parity.host_cache(w)
    rows = oracle.all_rows(c)
    qi, q = parity.host_queries(w, list(range(w.batch)))
    _, rbs = oracle.indexer(c, qi, w.s_qi, rows, token_scores=False)
    rsel = oracle.select(c, rows, rbs)
    nvis = np.array([(int(c.seq_lens[b]) - T + t) // 128 + 1 for b, t in rows])
    gsel = sel.cpu().numpy().reshape(len(rows), 4, 16)
    parity.check_selection(gsel, rsel, rbs, nvis, name)
    ref = oracle.attention(c, q, w.s_q, w.softmax_scale, rows, gsel)
    parity.check_output(out.reshape(len(rows), 64, 128), ref, name)
    # and the same as the ungrouped step
    out_u = torch.empty_like(out)
    sel_u = torch.empty_like(sel)
    msa.msa_decode(cache, seqs, w.qi, w.s_qi, w.q, w.s_q, w.softmax_scale, out_u, sel_u, ws)
    torch.cuda.synchronize()
    assert torch.equal(sel, sel_u)


def test_inconsistent_groups_are_reported():
    """A prefix longer than what every query of the group sees, and groups
    that do not cover the batch: reported as a device bounds error (the
    arrays are clamped, nothing is accessed outside the buffers)."""
    w = _workload("bad_groups", [3000, 3000], 1, [(2, 10)], {})
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    bs = torch.empty(w.batch, 1, 4, w.max_pages, device="cuda")
    for groups in ([(2, 30)], [(1, 10)]):
        ws = msa.alloc_workspace(seqs)
        g = msa.PrefixGroups.of(groups)
        msa.msa_indexer_score_grouped(cache, seqs, g, w.qi, w.s_qi, None, bs, ws)
        torch.cuda.synchronize()
        assert msa.msa_get_last_error(ws)[0] == msa.MSA_ERR_DEVICE_BOUNDS, groups


def test_grouped_requires_a_page_table():
    w = synth.make_workload("contig", 2, [3000, 3000], 1, paged=False, seed=5, device="cuda")
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    bs = torch.empty(w.batch, 1, 4, w.max_pages, device="cuda")
    with pytest.raises(msa.MsaError) as e:
        msa.msa_indexer_score_grouped(cache, seqs, msa.PrefixGroups.of([(2, 0)]), w.qi, w.s_qi, None, bs, ws)
    assert e.value.status == msa.MSA_ERR_INVALID_ARG
