"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Every comparison uses the tolerances stated in tests/parity.py.  Small cases
compare every output; the full-size workloads (the same launch configuration
the benchmark times) compare sampled sequences/tokens that the oracle can
compute one by one.
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_decode_b200 as msa
from block_sparse_attention_decode_b200 import build as msa_build
from block_sparse_attention_decode_b200 import synth
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="session", autouse=True)
def _lib():
    msa_build.build()
    msa.load()


def dev_workload(name, *args, **kw):
    return synth.make_workload(name, *args, device="cuda", **kw)


def run_decode(w, ws=None):
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    if ws is None:
        ws = msa.alloc_workspace(seqs)
    out = torch.empty(w.batch, w.q_tokens, 64, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(w.batch, w.q_tokens, 4, 16, dtype=torch.int32, device="cuda")
    msa.msa_decode(cache, seqs, w.qi, w.s_qi, w.q, w.s_q, w.softmax_scale, out, sel, ws)
    torch.cuda.synchronize()
    st, detail = msa.msa_get_last_error(ws)
    assert st == msa.MSA_OK, (st, detail)
    return out, sel


def run_indexer(w, token_level=True):
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    rows = w.batch * w.q_tokens
    ts = None
    if token_level:
        ts = torch.full((w.batch, w.q_tokens, 4, w.max_pages * 128), float("nan"), device="cuda")
    bs = torch.full((w.batch, w.q_tokens, 4, w.max_pages), float("nan"), device="cuda")
    msa.msa_indexer_score(cache, seqs, w.qi, w.s_qi, ts, bs, ws)
    torch.cuda.synchronize()
    assert msa.msa_get_last_error(ws)[0] == msa.MSA_OK
    return ts, bs


def nvis_of(c: oracle.Cache, rows):
    return np.array([(int(c.seq_lens[b]) - c.q_tokens + t) // 128 + 1 for b, t in rows])


def compare_decode(w, seq_ids=None, tokens=None, what=""):
    out, sel = run_decode(w)
    c, ids = parity.host_cache(w, seq_ids)
    qi, q = parity.host_queries(w, ids)
    T = w.q_tokens
    tokens = list(range(T)) if tokens is None else tokens
    rows = [(r, t) for r in range(len(ids)) for t in tokens]
    _, bs = oracle.indexer(c, qi, w.s_qi, rows, token_scores=False)
    ref_sel = oracle.select(c, rows, bs)
    gsel = np.stack([sel[ids[r], t].cpu().numpy() for r, t in rows])
    swaps = parity.check_selection(gsel, ref_sel, bs, nvis_of(c, rows), what)
    ref_out = oracle.attention(c, q, w.s_q, w.softmax_scale, rows, gsel)
    gout = torch.stack([out[ids[r], t] for r, t in rows])
    mx, mean = parity.check_output(gout, ref_out, what)
    return swaps, mx, mean


# ------------------------------------------------------------- formats -----
def test_nvfp4_table_bit_exact():
    out = torch.empty(256 * 16, dtype=torch.uint8, device="cuda")
    msa.msa_debug_nvfp4_table(out)
    got = out.cpu().numpy().reshape(256, 16)
    for s in range(256):
        if s in (0x7F, 0xFF):        # NaN scale bytes: never produced, not compared
            continue
        for c in range(16):
            ref = oracle.e4m3_round(oracle.e2m1(c) * oracle.e4m3(s))
            if oracle.e4m3(ref) == 0.0:          # +0 and -0 are the same value
                assert oracle.e4m3(int(got[s, c])) == 0.0, (hex(s), c)
            else:
                assert int(got[s, c]) == ref, (hex(s), c, hex(got[s, c]), hex(ref))


# ------------------------------------------------------------- indexer -----
SMALL = [
    ("t1_paged_ragged", dict(batch=3, seq_lens=[300, 2049, 5000], q_tokens=1, paged=True, seed=21)),
    ("t2_contig", dict(batch=2, seq_lens=[4096, 1500], q_tokens=2, paged=False, seed=22)),
    ("t8_paged", dict(batch=2, seq_lens=[3000, 9000], q_tokens=8, paged=True, seed=23)),
    ("t8_boundary", dict(batch=2, seq_lens=[2052, 2176], q_tokens=8, paged=True, seed=24)),
    ("t3_odd", dict(batch=3, seq_lens=[3, 130, 4100], q_tokens=3, paged=True, seed=25)),
    ("fp8idx", dict(batch=2, seq_lens=[2500, 6000], q_tokens=1, paged=False, seed=26, idx_fp8=True)),
    ("t5_fp8idx", dict(batch=2, seq_lens=[2100, 2900], q_tokens=5, paged=True, seed=27, idx_fp8=True)),
    ("saturating_scales", dict(batch=2, seq_lens=[2300, 700], q_tokens=1, paged=True, seed=28,
                               scale_floor_byte=0x68)),
    ("planted", dict(batch=2, seq_lens=[8192, 8192], q_tokens=1, paged=False, seed=29,
                     plant_every=8)),
    ("neg_scales", dict(batch=2, seq_lens=[5000, 2600], q_tokens=4, paged=True, seed=30,
                        neg_scale_frac=0.05)),
]

# NVFP4 index keys scored at their exact value (MSA_IDX_NVFP4_EXACT): query
# tiles of 8, 32 and 256 index queries, signed scales, ragged tails.
EXACT = [
    ("t1_exact", dict(batch=3, seq_lens=[300, 2049, 5000], q_tokens=1, paged=True, seed=32,
                      idx_exact=True)),
    ("t8_exact", dict(batch=2, seq_lens=[3000, 9000], q_tokens=8, paged=True, seed=33,
                      idx_exact=True)),
    ("neg_scales_exact", dict(batch=2, seq_lens=[5000, 2600], q_tokens=4, paged=True, seed=34,
                              neg_scale_frac=0.05, idx_exact=True)),
    ("t64_exact", dict(batch=1, seq_lens=[4000], q_tokens=64, paged=True, seed=35,
                       idx_exact=True)),
]


@pytest.mark.parametrize("name,kw", SMALL + EXACT, ids=[s[0] for s in SMALL + EXACT])
def test_indexer_scores(name, kw):
    w = dev_workload(name, **kw)
    ts, bs = run_indexer(w)
    c, _ = parity.host_cache(w)
    rows = oracle.all_rows(c)
    rts, rbs = oracle.indexer(c, w.qi.cpu().numpy(), w.s_qi, rows, ctx_cap=w.max_pages * 128)
    gts = ts.cpu().numpy().reshape(len(rows), 4, -1)
    gbs = bs.cpu().numpy().reshape(len(rows), 4, -1)
    for r, (b, t) in enumerate(rows):
        L = int(c.seq_lens[b])
        nblk = (L + 127) // 128
        pos = L - w.q_tokens + t
        # token scores: visible keys scored, the rest of the written blocks -inf
        ref_t = np.full((4, nblk * 128), -np.inf)
        ref_t[:, :pos + 1] = rts[r, :, :pos + 1]
        parity.check_scores(gts[r, :, :nblk * 128], ref_t, "%s token scores row %d" % (name, r))
        parity.check_scores(gbs[r, :, :nblk], rbs[r, :, :nblk], "%s block scores row %d" % (name, r))


def test_exact_mode_is_not_rerounded():
    """The exact-mode scores sit on the unrounded oracle, far (relative to the
    score tolerance) from the E4M3 re-rounded one, and the two GPU modes differ."""
    w = dev_workload("exact_vs_rr", 2, [3000, 9000], 8, paged=True, seed=33, idx_exact=True)
    ts, _ = run_indexer(w)
    ts_rr, _ = run_indexer(synth.Workload(**{**w.__dict__, "idx_exact": False}))
    c, _ = parity.host_cache(w)
    rows = oracle.all_rows(c)
    c.idx_exact = False
    rts_rr, _ = oracle.indexer(c, w.qi.cpu().numpy(), w.s_qi, rows, ctx_cap=w.max_pages * 128)
    g = ts.cpu().numpy().reshape(len(rows), 4, -1)
    b, t = rows[0]
    pos = int(c.seq_lens[b]) - w.q_tokens + t
    with pytest.raises(AssertionError):
        parity.check_scores(g[0, :, :pos + 1], rts_rr[0, :, :pos + 1], "exact vs re-rounded")
    assert not torch.equal(ts, ts_rr)


def test_block_scores_independent_of_batch_composition():
    """A sequence scored alone and inside a batch (different CTA slices of
    the page list) gives bit-identical block scores."""
    w = dev_workload("compose", 4, [7000, 40000, 300, 12345], 2, paged=True, seed=31)
    _, bs_all = run_indexer(w, token_level=False)
    for b in (1, 3):
        w1 = synth.Workload(**{**w.__dict__, "batch": 1, "seq_lens": w.seq_lens[b:b + 1].clone(),
                               "page_table": w.page_table[b:b + 1].clone(), "qi": w.qi[b:b + 1].clone(),
                               "q": w.q[b:b + 1].clone()})
        _, bs1 = run_indexer(w1, token_level=False)
        nb = (int(w.seq_lens[b]) + 127) // 128
        assert torch.equal(bs1[0, :, :, :nb], bs_all[b, :, :, :nb])


# ------------------------------------------------------------- top-k -------
def _topk_case(scores64: np.ndarray, lens, T):
    """GPU top-k on fp32 scores vs the oracle's selection of the SAME fp32
    values (so both rank identical numbers): must match exactly."""
    B = len(lens)
    max_pages = scores64.shape[-1]
    s32 = scores64.astype(np.float32)
    seqs = msa.Seqs(torch.tensor(lens, dtype=torch.int32, device="cuda"), T, max_pages)
    ws = msa.alloc_workspace(seqs)
    sel = torch.empty(B, T, 4, 16, dtype=torch.int32, device="cuda")
    msa.msa_block_maxpool_topk(torch.from_numpy(s32).cuda(), False, seqs, sel, ws)
    torch.cuda.synchronize()
    dummy = np.zeros((1, 4, 128, 64), np.uint8)
    c = oracle.Cache(idx_data=np.zeros((1, 128, 64), np.uint8), idx_scale=np.zeros((1, 128, 8), np.uint8),
                     k_data=dummy, k_scale=np.zeros((1, 4, 128, 8), np.uint8), v_data=dummy,
                     v_scale=np.zeros((1, 4, 128, 8), np.uint8), s_idx=1, s_k=1, s_v=1,
                     page_table=None, max_pages=max_pages, seq_lens=np.array(lens, np.int32),
                     q_tokens=T)
    rows = oracle.all_rows(c)
    ref = oracle.select(c, rows, s32.astype(np.float64).reshape(len(rows), 4, max_pages))
    np.testing.assert_array_equal(sel.cpu().numpy().reshape(len(rows), 4, 16), ref)


def test_topk_exact_random():
    rng = np.random.default_rng(41)
    lens = [100, 2048, 2049, 16 * 128 + 5, 300000 // 3, 262144]
    mp = 2048
    T = 2
    s = rng.normal(size=(len(lens), T, 4, mp))
    _topk_case(s, lens, T)


def test_topk_exact_heavy_ties_and_signs():
    rng = np.random.default_rng(42)
    lens = [5000, 70000, 2177]
    mp = 600
    T = 3
    s = rng.integers(-3, 3, size=(len(lens), T, 4, mp)).astype(np.float64)
    s[0, 0, 0, :] = 0.0                      # all equal: lowest ids win
    s[1, 1, 2, ::7] = -np.inf                # -inf candidates
    s[2, 2, 1, :] = -0.0
    _topk_case(s, lens, T)


def test_topk_token_level_input():
    w = dev_workload("toklevel", 2, [3000, 2600], 2, paged=True, seed=43)
    c, _ = parity.host_cache(w)
    rows = oracle.all_rows(c)
    rts, _ = oracle.indexer(c, w.qi.cpu().numpy(), w.s_qi, rows, ctx_cap=w.max_pages * 128)
    ts32 = np.where(np.isnan(rts), -np.inf, rts).astype(np.float32)
    seqs = msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    sel = torch.empty(w.batch, w.q_tokens, 4, 16, dtype=torch.int32, device="cuda")
    msa.msa_block_maxpool_topk(torch.from_numpy(ts32).cuda(), True, seqs, sel, ws)
    torch.cuda.synchronize()
    # oracle selection over the max-pool of the same fp32 token scores
    bs = np.full((len(rows), 4, w.max_pages), -np.inf)
    for r, (b, t) in enumerate(rows):
        pos = int(c.seq_lens[b]) - w.q_tokens + t
        for i in range(pos // 128 + 1):
            bs[r, :, i] = ts32[r, :, i * 128: min(pos + 1, i * 128 + 128)].astype(np.float64).max(axis=1)
    ref = oracle.select(c, rows, bs)
    np.testing.assert_array_equal(sel.cpu().numpy().reshape(len(rows), 4, 16), ref)


# ----------------------------------------------------------- attention -----
ATT_CASES = SMALL[:5] + SMALL[-1:]


@pytest.mark.parametrize("name,kw", ATT_CASES, ids=[s[0] for s in ATT_CASES])
def test_attention_given_oracle_selection(name, kw):
    w = dev_workload(name, **kw)
    c, _ = parity.host_cache(w)
    rows = oracle.all_rows(c)
    _, bs = oracle.indexer(c, w.qi.cpu().numpy(), w.s_qi, rows, token_scores=False)
    ref_sel = oracle.select(c, rows, bs)
    ref_out = oracle.attention(c, w.q.cpu().numpy(), w.s_q, w.softmax_scale, rows, ref_sel)
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    out = torch.empty(w.batch, w.q_tokens, 64, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.from_numpy(ref_sel.reshape(w.batch, w.q_tokens, 4, 16)).cuda()
    msa.msa_sparse_attn_decode(cache, seqs, w.q, w.s_q, sel, w.softmax_scale, out, ws)
    torch.cuda.synchronize()
    assert msa.msa_get_last_error(ws)[0] == msa.MSA_OK
    parity.check_output(out.reshape(len(rows), 64, 128), ref_out, name)


# ------------------------------------------------------------- decode ------
@pytest.mark.parametrize("name,kw", SMALL + EXACT, ids=[s[0] for s in SMALL + EXACT])
def test_decode_small(name, kw):
    w = dev_workload(name, **kw)
    compare_decode(w, what=name)


def test_dense_when_at_most_16_blocks():
    """<= 16 visible blocks: every block selected (dense attention)."""
    w = dev_workload("dense", 3, [2048, 1, 900], 1, paged=True, seed=51)
    out, sel = run_decode(w)
    s = sel.cpu().numpy()
    for b, L in enumerate([2048, 1, 900]):
        nb = (L - 1) // 128 + 1
        for g in range(4):
            assert list(s[b, 0, g]) == list(range(nb)) + [-1] * (16 - nb)
    compare_decode(w, what="dense")


def test_paged_equals_contiguous_bitwise():
    wc = dev_workload("contig", 2, [9000, 20000], 2, paged=False, seed=52)
    perm = torch.randperm(wc.num_pages, generator=torch.Generator().manual_seed(5)).to(torch.int32)
    inv = torch.argsort(perm).cuda()
    pool = lambda t: None if t is None else t[inv].contiguous()
    wp = synth.Workload(**{**wc.__dict__, "page_table": perm.view(2, wc.max_pages).cuda(),
                           "idx_data": pool(wc.idx_data), "idx_scale": pool(wc.idx_scale),
                           "k_data": pool(wc.k_data), "k_scale": pool(wc.k_scale),
                           "v_data": pool(wc.v_data), "v_scale": pool(wc.v_scale)})
    oc, sc = run_decode(wc)
    op, sp = run_decode(wp)
    assert torch.equal(sc, sp)
    assert torch.equal(oc, op)


def test_repeat_calls_reuse_workspace():
    w = dev_workload("repeat", 3, [20000, 33000, 4000], 1, paged=True, seed=53)
    seqs = msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    o1, s1 = run_decode(w, ws)
    o2, s2 = run_decode(w, ws)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
    # the indexer's and the attention's work counters (workspace header
    # bytes 64..79) are back at 0
    assert ws[64:80].view(torch.int32).tolist() == [0, 0, 0, 0]


def test_split_k_with_empty_slices_repeated():
    """Few rows (8 sequences x 1 token x 4 groups): the attention splits each
    row's 16 selected blocks into 16 one-block slices merged through fp32
    partials, and a slice past a short sequence's last visible block is an
    empty item, which passes through the pipeline without a load or an MMA.
    Twenty calls on one workspace give the same bits (the row counters go
    back to 0 and no item's hand-offs race ahead of another's), and the first
    matches the oracle."""
    lens = [300, 700, 1025, 130, 5000, 2000, 900, 64]
    w = dev_workload("empty_slices", len(lens), lens, 1, paged=True, seed=54)
    seqs = msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    o1, s1 = run_decode(w, ws)
    for _ in range(19):
        o2, s2 = run_decode(w, ws)
        assert torch.equal(s1, s2)
        assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    compare_decode(w, what="split-K with empty slices")


# batches whose (sequence, token, group) rows take 8, 4 and 2 slices each (rows x
# slices >= 4 x 148), short sequences among long ones: empty and partial slices
SPLIT_CASES = [(8, 19), (4, 37), (2, 74)]


@pytest.mark.parametrize("splits,batch", SPLIT_CASES, ids=["splits%d" % s for s, _ in SPLIT_CASES])
def test_split_counts_with_empty_slices(splits, batch):
    """Each split count of the attention's split-K on one token per sequence:
    the rows' outputs against the oracle over the GPU's own selection (on
    every fourth sequence, all lengths represented), and two calls on one
    workspace bit-identical."""
    rows = batch * 4
    assert rows * splits >= 4 * 148 and (splits == 16 or rows * splits // 2 < 4 * 148)
    cycle = [300, 700, 1025, 130, 5000, 2000, 900, 64, 9000, 16000, 2049]
    lens = [cycle[i % len(cycle)] for i in range(batch)]
    w = dev_workload("splits%d" % splits, batch, lens, 1, paged=True, seed=55 + splits)
    seqs = msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    o1, s1 = run_decode(w, ws)
    o2, s2 = run_decode(w, ws)
    assert torch.equal(s1, s2)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    compare_decode(w, seq_ids=list(range(0, batch, 4)), what="split-K x%d" % splits)


# ---------------------------------------------------------- boundaries -----
def test_bad_page_id_sets_device_flag_and_context_survives():
    w = dev_workload("badpage", 2, [5000, 3000], 1, paged=True, seed=61)
    bad_pt = w.page_table.clone()
    bad_pt[1, 3] = w.num_pages + 7           # out of the pool: must be skipped + reported
    wb = synth.Workload(**{**w.__dict__, "page_table": bad_pt})
    cache, seqs = msa.cache_of(wb), msa.seqs_of(wb)
    ws = msa.alloc_workspace(seqs)
    out = torch.empty(2, 1, 64, 128, dtype=torch.bfloat16, device="cuda")
    msa.msa_decode(cache, seqs, wb.qi, wb.s_qi, wb.q, wb.s_q, wb.softmax_scale, out, None, ws)
    st, detail = msa.msa_get_last_error(ws)
    assert st == msa.MSA_ERR_DEVICE_BOUNDS and detail == w.num_pages + 7
    assert msa.msa_get_last_error(ws)[0] == msa.MSA_OK      # cleared
    run_decode(w)                                           # context still usable


def test_bad_selected_block_sets_device_flag():
    w = dev_workload("badsel", 1, [5000], 1, paged=True, seed=62)
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    sel = torch.full((1, 1, 4, 16), -1, dtype=torch.int32, device="cuda")
    sel[0, 0, :, 0] = 39                      # visible blocks are 0..39
    sel[0, 0, 2, 1] = 40                      # not visible: error, skipped
    out = torch.empty(1, 1, 64, 128, dtype=torch.bfloat16, device="cuda")
    msa.msa_sparse_attn_decode(cache, seqs, w.q, w.s_q, sel, w.softmax_scale, out, ws)
    st, detail = msa.msa_get_last_error(ws)
    assert st == msa.MSA_ERR_DEVICE_BOUNDS and detail == 40


def test_host_checks_launch_nothing():
    w = dev_workload("hostchk", 1, [500], 1, paged=False, seed=63)
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    out = torch.empty(1, 1, 64, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(msa.MsaError) as e:
        msa.msa_decode(cache, seqs, w.qi, -1.0, w.q, w.s_q, w.softmax_scale, out, None, ws)
    assert e.value.status == msa.MSA_ERR_INVALID_ARG
    with pytest.raises(msa.MsaError) as e:
        msa.msa_decode(cache, seqs, w.qi, w.s_qi, w.q, w.s_q, w.softmax_scale, out, None, ws[:64])
    assert e.value.status == msa.MSA_ERR_WORKSPACE
