"""Property pins of the oracle over random small inputs (hypothesis):

  * selection: ascending distinct ids, the query's latest block always in,
    min(visible blocks, 16) of them, every id visible, and no unselected
    visible block ranked above a selected one ([post, "MSA primer"]);
  * attention: each output element lies inside the range of the selected
    visible V values of its group times s_v (a softmax is a convex weight);
  * exact index mode: scores are linear in the index-key scale s_idx.
"""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle
from block_sparse_attention_decode_b200 import synth
from tests import parity

SETTINGS = dict(max_examples=12, deadline=None)


def _case(draw_lens, T, seed, paged, exact=False):
    w = synth.make_workload("prop", len(draw_lens), draw_lens, T, paged=paged, seed=seed,
                            idx_exact=exact)
    c, _ = parity.host_cache(w)
    return w, c, oracle.all_rows(c)


lens_st = st.lists(st.integers(min_value=8, max_value=3000), min_size=1, max_size=3)


@settings(**SETTINGS)
@given(lens=lens_st, T=st.integers(1, 8), seed=st.integers(0, 10_000), paged=st.booleans())
def test_selection_properties(lens, T, seed, paged):
    lens = [max(L, T) for L in lens]
    w, c, rows = _case(lens, T, seed, paged)
    _, bs = oracle.indexer(c, w.qi.numpy(), w.s_qi, rows, token_scores=False)
    sel = oracle.select(c, rows, bs)
    for r, (b, t) in enumerate(rows):
        pos = int(c.seq_lens[b]) - T + t
        latest, nvis = pos // 128, pos // 128 + 1
        for g in range(4):
            ids = [int(x) for x in sel[r, g] if x >= 0]
            assert ids == sorted(set(ids)) and len(ids) == min(nvis, 16)
            assert latest in ids and all(0 <= i <= latest for i in ids)
            assert all(x == -1 for x in sel[r, g, len(ids):])
            others = [i for i in ids if i != latest]
            rest = [i for i in range(latest) if i not in ids]
            if others and rest:
                S = bs[r, g]
                worst_in = min(others, key=lambda i: (S[i], -i))
                best_out = max(rest, key=lambda i: (S[i], -i))
                assert (S[worst_in], -worst_in) > (S[best_out], -best_out)


@settings(**SETTINGS)
@given(lens=lens_st, T=st.integers(1, 4), seed=st.integers(0, 10_000))
def test_attention_inside_the_value_range(lens, T, seed):
    lens = [max(L, T) for L in lens]
    w, c, rows = _case(lens, T, seed, True)
    _, bs = oracle.indexer(c, w.qi.numpy(), w.s_qi, rows, token_scores=False)
    sel = oracle.select(c, rows, bs)
    out = oracle.attention(c, w.q.numpy(), w.s_q, w.softmax_scale, rows, sel)
    for r, (b, t) in enumerate(rows):
        pos = int(c.seq_lens[b]) - T + t
        for g in range(4):
            keys = [j for blk in sel[r, g] if blk >= 0
                    for j in range(blk * 128, min(blk * 128 + 128, pos + 1))]
            vals = []
            for j in keys:
                p = int(c.page_table[b, j // 128])
                vals.append(oracle.decode_nvfp4_row(c.v_data[p, g, j % 128],
                                                    c.v_scale[p, g, j % 128]))
            vals = np.array(vals) * c.s_v
            lo, hi = vals.min(axis=0), vals.max(axis=0)
            o = out[r, 16 * g:16 * g + 16]                   # the group's 16 heads
            slack = 2.0 ** -8 * np.maximum(np.abs(lo), np.abs(hi)) + 1e-12   # bf16 rounding
            assert np.all(o >= lo - slack) and np.all(o <= hi + slack)


@settings(**SETTINGS)
@given(L=st.integers(1, 2000), seed=st.integers(0, 10_000), k=st.sampled_from([0.5, 2.0, 3.0]))
def test_exact_scores_linear_in_index_scale(L, seed, k):
    w, c, rows = _case([L], 1, seed, False, exact=True)
    ts1, _ = oracle.indexer(c, w.qi.numpy(), w.s_qi, rows)
    c.s_idx = c.s_idx * k
    ts2, _ = oracle.indexer(c, w.qi.numpy(), w.s_qi, rows)
    np.testing.assert_allclose(ts2[:, :, :L], k * ts1[:, :, :L], rtol=1e-12, atol=0)
