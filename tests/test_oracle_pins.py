"""Pins for the oracle's steps (CPU only), each against something other than
the oracle itself: library routines (torch.matmul, max_pool1d, numpy lexsort,
scaled_dot_product_attention -- on bytes decoded by torch's float8 cast),
closed forms, invariants and brute force on tiny contexts.

Method: vLLM 為 MiniMax-M3.1-Flash 提供 Day-0 支援 (hot.atechcom.net),
"MSA primer" (indexer, max-pool, top-16 with the latest block kept, <=2,048
keys, exact attention over the selected blocks; Figure 1 caption: every query
head of a group attends over its group's blocks).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_decode_b200 import synth
from tests import torch_ref


def to_cache(w) -> oracle.Cache:
    n = lambda t: None if t is None else t.cpu().numpy()
    return oracle.Cache(idx_data=n(w.idx_data), idx_scale=n(w.idx_scale), k_data=n(w.k_data),
                        k_scale=n(w.k_scale), v_data=n(w.v_data), v_scale=n(w.v_scale),
                        s_idx=w.s_idx, s_k=w.s_k, s_v=w.s_v, page_table=n(w.page_table),
                        max_pages=w.max_pages, seq_lens=n(w.seq_lens), q_tokens=w.q_tokens)


@pytest.fixture(scope="module")
def small():
    # 3 sequences, 2 query tokens, partial last blocks, a paged shuffled cache;
    # lengths straddle the 16-block boundary (dense vs sparse).
    return synth.make_workload("pin_small", 3, [300, 2049, 2600], 2, paged=True, seed=11)


@pytest.fixture(scope="module")
def small_rows(small):
    return oracle.all_rows(to_cache(small))


# ------------------------------------------------------------- indexer -----
def test_token_scores_vs_torch_matmul(small, small_rows):
    c = to_cache(small)
    sc, _ = oracle.indexer(c, small.qi.numpy(), small.s_qi, small_rows)
    for r, (b, t) in enumerate(small_rows):
        ref = torch_ref.token_scores(small, b, t).numpy()
        n = ref.shape[1]
        np.testing.assert_allclose(sc[r, :, :n], ref, rtol=1e-12, atol=1e-12)
        assert np.isnan(sc[r, :, n:]).all()          # positions after the query: untouched


def test_fp8_index_keys_vs_torch_matmul():
    w = synth.make_workload("pin_fp8", 2, [700, 140], 1, paged=False, seed=12, idx_fp8=True)
    c = to_cache(w)
    rows = oracle.all_rows(c)
    sc, bs = oracle.indexer(c, w.qi.numpy(), w.s_qi, rows)
    for r, (b, t) in enumerate(rows):
        ref = torch_ref.token_scores(w, b, t).numpy()
        np.testing.assert_allclose(sc[r, :, :ref.shape[1]], ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(bs[r], torch_ref.block_scores(w, b, t).numpy(), rtol=1e-12)


def test_unit_query_reads_one_key_element(small):
    """qi = e_d for group g: the score of token j equals s_qi*s_idx*k_j[d] --
    pins the dimension, nibble, scale and page indexing."""
    w = small
    qi = np.zeros_like(w.qi.numpy())
    dims = [0, 1, 17, 64, 127]
    one = 0x38  # E4M3 1.0
    for g, d in enumerate(dims[:4]):
        qi[:, :, g, d] = one
    c = to_cache(w)
    rows = oracle.all_rows(c)
    sc, _ = oracle.indexer(c, qi, 1.0, rows)
    for r, (b, t) in enumerate(rows):
        K = torch_ref.index_keys(w, b).numpy()
        pos = int(w.seq_lens[b]) - w.q_tokens + t
        for g, d in enumerate(dims[:4]):
            np.testing.assert_array_equal(sc[r, g, :pos + 1], K[:pos + 1, d])


def test_block_scores_vs_max_pool(small, small_rows):
    c = to_cache(small)
    _, bs = oracle.indexer(c, small.qi.numpy(), small.s_qi, small_rows, token_scores=False)
    for r, (b, t) in enumerate(small_rows):
        np.testing.assert_allclose(bs[r], torch_ref.block_scores(small, b, t).numpy(),
                                   rtol=1e-12, atol=1e-12)


def test_planted_key_wins_its_block():
    """A key far above the rest at logical position j puts block j//128 on top."""
    w = synth.make_workload("pin_plant", 1, [5000], 1, paged=True, seed=13)
    j = 3333
    page = int(w.page_table[0, j // 128])
    w.idx_data[page, j % 128] = 0x77           # all codes +6
    w.idx_scale[page, j % 128] = 0x60          # scale 32: 192 per element, ~29 sigma
    qi = w.qi.clone()
    qi[0, 0, 1] = 0x38                         # group 1 query = all ones
    c = to_cache(w)
    _, bs = oracle.indexer(c, qi.numpy(), w.s_qi, [(0, 0)], token_scores=False)
    assert int(np.argmax(bs[0, 1])) == j // 128
    sel = oracle.select(c, [(0, 0)], bs)
    assert j // 128 in sel[0, 1]


def test_page_table_invariance():
    """The same logical cache, contiguous and behind a shuffled page table."""
    wc = synth.make_workload("pin_contig", 2, [2500, 1800], 1, paged=False, seed=14)
    perm = np.random.default_rng(3).permutation(wc.num_pages).astype(np.int32)
    inv = np.argsort(perm)
    cc = to_cache(wc)
    pool = lambda a: None if a is None else np.ascontiguousarray(a[inv])
    # physical page perm[k] holds logical page k
    cp = oracle.Cache(idx_data=pool(cc.idx_data), idx_scale=pool(cc.idx_scale),
                      k_data=pool(cc.k_data), k_scale=pool(cc.k_scale), v_data=pool(cc.v_data),
                      v_scale=pool(cc.v_scale), s_idx=cc.s_idx, s_k=cc.s_k, s_v=cc.s_v,
                      page_table=perm.reshape(2, wc.max_pages), max_pages=cc.max_pages,
                      seq_lens=cc.seq_lens, q_tokens=cc.q_tokens)
    rows = oracle.all_rows(cc)
    a = oracle.decode(cc, wc.qi.numpy(), wc.s_qi, wc.q.numpy(), wc.s_q, wc.softmax_scale, rows)
    b = oracle.decode(cp, wc.qi.numpy(), wc.s_qi, wc.q.numpy(), wc.s_q, wc.softmax_scale, rows)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_token_permutation_inside_block_keeps_block_scores():
    w = synth.make_workload("pin_perm", 1, [1280], 1, paged=False, seed=15)
    c = to_cache(w)
    _, bs0 = oracle.indexer(c, w.qi.numpy(), w.s_qi, [(0, 0)], token_scores=False)
    rng = np.random.default_rng(1)
    c2 = to_cache(w)
    for p in range(w.num_pages - 1):   # full blocks only (last block holds the query)
        perm = rng.permutation(128)
        c2.idx_data[p] = c2.idx_data[p][perm]
        c2.idx_scale[p] = c2.idx_scale[p][perm]
    _, bs1 = oracle.indexer(c2, w.qi.numpy(), w.s_qi, [(0, 0)], token_scores=False)
    assert np.array_equal(bs0, bs1)


# ----------------------------------------------------------- selection -----
def test_selection_vs_library_sort_and_definition(small, small_rows):
    c = to_cache(small)
    _, bs = oracle.indexer(c, small.qi.numpy(), small.s_qi, small_rows, token_scores=False)
    sel = oracle.select(c, small_rows, bs)
    for r, (b, t) in enumerate(small_rows):
        pos = int(small.seq_lens[b]) - small.q_tokens + t
        nb = pos // 128 + 1
        for g in range(4):
            s = [int(x) for x in sel[r, g] if x >= 0]
            assert s == torch_ref.select_by_sort(bs[r, g], nb)
            assert len(s) == min(nb, 16) and s == sorted(s) and (nb - 1) in s
            assert all(x == -1 for x in sel[r, g, len(s):])
            assert sum(min(128, pos + 1 - 128 * i) for i in s) <= 2048


def test_selection_definition_brute_force():
    """Random block scores with many ties: every chosen block (other than the
    latest) ranks ahead of every block left out, by (score desc, id asc)."""
    rng = np.random.default_rng(5)
    for nb in (1, 5, 16, 17, 18, 40, 200):
        L = nb * 128
        c = oracle.Cache(idx_data=np.zeros((nb, 128, 64), np.uint8),
                         idx_scale=np.zeros((nb, 128, 8), np.uint8),
                         k_data=np.zeros((nb, 4, 128, 64), np.uint8),
                         k_scale=np.zeros((nb, 4, 128, 8), np.uint8),
                         v_data=np.zeros((nb, 4, 128, 64), np.uint8),
                         v_scale=np.zeros((nb, 4, 128, 8), np.uint8),
                         s_idx=1, s_k=1, s_v=1, page_table=None, max_pages=nb,
                         seq_lens=np.array([L], np.int32), q_tokens=1)
        bs = rng.integers(0, 6, (1, 4, nb)).astype(np.float64)   # heavy ties
        sel = oracle.select(c, [(0, 0)], bs)
        for g in range(4):
            s = set(int(x) for x in sel[0, g] if x >= 0)
            assert len(s) == min(nb, 16) and (nb - 1) in s
            key = lambda i: (-bs[0, g, i], i)
            inside = [i for i in s if i != nb - 1]
            outside = [i for i in range(nb - 1) if i not in s]
            if inside and outside:
                assert max(key(i) for i in inside) < min(key(i) for i in outside)


def test_selection_invariant_to_positive_index_scale(small, small_rows):
    c = to_cache(small)
    _, bs = oracle.indexer(c, small.qi.numpy(), small.s_qi, small_rows, token_scores=False)
    c.s_idx = small.s_idx * 3.7
    _, bs2 = oracle.indexer(c, small.qi.numpy(), small.s_qi, small_rows, token_scores=False)
    assert np.array_equal(oracle.select(c, small_rows, bs), oracle.select(c, small_rows, bs2))


def test_split_then_merge_equals_global():
    """Candidates split into context shards; merging each shard's local
    top-15 gives the global top-15 (the exactness the indexer decode context
    parallelism relies on, "NVFP4 indexer DCP")."""
    rng = np.random.default_rng(9)
    nb = 301
    scores = np.round(rng.normal(size=nb), 2)   # rounded: ties across shards
    glob = torch_ref.select_by_sort(scores, nb)
    for nshard in (2, 3, 7):
        bounds = np.linspace(0, nb - 1, nshard + 1).astype(int)
        cand = []
        for a, b in zip(bounds[:-1], bounds[1:]):
            ids = np.arange(a, b)
            order = np.lexsort((ids, -scores[a:b]))[:15]
            cand.extend(ids[order])
        cand = np.array(sorted(cand))
        order = np.lexsort((cand, -scores[cand]))[:15]
        assert sorted(list(cand[order]) + [nb - 1]) == glob


# ----------------------------------------------------------- attention -----
def test_attention_vs_sdpa_over_selection(small, small_rows):
    c = to_cache(small)
    bs, sel, out = oracle.decode(c, small.qi.numpy(), small.s_qi, small.q.numpy(), small.s_q,
                                 small.softmax_scale, small_rows)
    for r, (b, t) in enumerate(small_rows):
        ref = torch_ref.attention_sdpa(small, b, t, sel[r], small.softmax_scale).numpy()
        np.testing.assert_allclose(out[r], ref, rtol=1e-9, atol=1e-12)


def test_dense_equality_when_at_most_16_blocks():
    """Context <= 16 blocks: every block selected, so the path equals dense
    causal attention over all keys (SDPA with is_causal-like mask)."""
    w = synth.make_workload("pin_dense", 2, [2048, 1500], 3, paged=True, seed=16)
    c = to_cache(w)
    rows = oracle.all_rows(c)
    bs, sel, out = oracle.decode(c, w.qi.numpy(), w.s_qi, w.q.numpy(), w.s_q,
                                 w.softmax_scale, rows)
    for r, (b, t) in enumerate(rows):
        L = int(w.seq_lens[b])
        pos = L - w.q_tokens + t
        K, V = torch_ref.kv(w, b, "k")[:, : pos + 1], torch_ref.kv(w, b, "v")[:, : pos + 1]
        q = torch_ref.e4m3_to_f64(w.q[b, t]) * w.s_q
        Kh = K.repeat_interleave(16, dim=0)       # head h uses KV head h//16
        Vh = V.repeat_interleave(16, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q.unsqueeze(1), Kh, Vh, scale=w.softmax_scale)[:, 0]
        np.testing.assert_allclose(out[r], ref.numpy(), rtol=1e-9, atol=1e-12)
        assert all(list(sel[r, g][sel[r, g] >= 0]) == list(range(pos // 128 + 1))
                   for g in range(4))


def test_constant_v_gives_that_vector():
    w = synth.make_workload("pin_constv", 1, [3000], 1, paged=False, seed=17)
    w.v_data[:] = 0x53     # codes 3 (1.5) / 5 (3.0) alternating
    w.v_scale[:] = 0x38    # scale 1.0
    c = to_cache(w)
    _, _, out = oracle.decode(c, w.qi.numpy(), w.s_qi, w.q.numpy(), w.s_q, w.softmax_scale,
                              [(0, 0)])
    expect = np.tile([1.5, 3.0], 64) * w.s_v
    np.testing.assert_allclose(out[0], np.broadcast_to(expect, (64, 128)), rtol=1e-12)


def test_one_dominant_key_returns_its_value():
    w = synth.make_workload("pin_dom", 1, [2100], 1, paged=False, seed=18)
    j = 2099 - 50
    w.q[:] = 0x38                                   # q = all ones (1.0 * s_q)
    w.k_data[:, :, :, :] = 0x00
    w.k_data[j // 128, :, j % 128, :] = 0x77        # key j = all +6 on every head
    w.k_scale[:] = 0x38
    c = to_cache(w)
    _, _, out = oracle.decode(c, w.qi.numpy(), w.s_qi, w.q.numpy(), 64.0, 1.0, [(0, 0)])
    V = torch_ref.kv(w, 0, "v")[:, j].numpy()       # [4][128]
    for h in range(64):
        np.testing.assert_allclose(out[0, h], V[h // 16], rtol=1e-9, atol=1e-9)


def test_scales_enter_linearly():
    """Doubling s_v doubles the output; multiplying s_q by a and dividing the
    softmax scale by a leaves it unchanged."""
    w = synth.make_workload("pin_lin", 1, [2300], 1, paged=False, seed=19)
    c = to_cache(w)
    rows = [(0, 0)]
    _, sel, out = oracle.decode(c, w.qi.numpy(), w.s_qi, w.q.numpy(), w.s_q, w.softmax_scale, rows)
    c.s_v = w.s_v * 2
    out2 = oracle.attention(c, w.q.numpy(), w.s_q, w.softmax_scale, rows, sel)
    np.testing.assert_allclose(out2, 2 * out, rtol=1e-12)
    c.s_v = w.s_v
    out3 = oracle.attention(c, w.q.numpy(), w.s_q * 4, w.softmax_scale / 4, rows, sel)
    np.testing.assert_allclose(out3, out, rtol=1e-12, atol=1e-15)
