"""GPU parity of msa_kv_insert against the oracle's cache insert: the whole
cache must be byte-identical after inserting the new tokens (codes, scales,
FP8 index keys), including midpoint ties, zero and saturating blocks; a page
outside the pool is reported and its rows skipped."""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_decode_b200 as msa
from block_sparse_attention_decode_b200 import synth

pytestmark = pytest.mark.gpu


def _inputs(w, seed, scale=1.0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    B, T = w.batch, w.q_tokens
    mk = lambda *s: (torch.randn(*s, generator=g, device="cuda") * scale).to(torch.bfloat16)
    return mk(B, T, 4, 128), mk(B, T, 4, 128), mk(B, T, 128)


def _oracle_insert(w, k, v, ix):
    """The oracle's insert on a host copy of the whole cache, same page layout."""
    h = lambda t: None if t is None else t.cpu().numpy().copy()
    c = oracle.Cache(idx_data=h(w.idx_data), idx_scale=h(w.idx_scale), k_data=h(w.k_data),
                     k_scale=h(w.k_scale), v_data=h(w.v_data), v_scale=h(w.v_scale),
                     s_idx=w.s_idx, s_k=w.s_k, s_v=w.s_v,
                     page_table=h(w.page_table), max_pages=w.max_pages,
                     seq_lens=np.ascontiguousarray(w.seq_lens.cpu().numpy(), dtype=np.int32),
                     q_tokens=w.q_tokens)
    rc = oracle.kv_insert(c, k.float().cpu().numpy(), v.float().cpu().numpy(), ix.float().cpu().numpy())
    assert rc == 0
    return c


def _gpu_insert(w, k, v, ix):
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    msa.msa_kv_insert(cache, seqs, k, v, ix, ws)
    torch.cuda.synchronize()
    return msa.msa_get_last_error(ws)


def _same(w, c):
    for name in ("k_data", "k_scale", "v_data", "v_scale", "idx_data", "idx_scale"):
        got = getattr(w, name)
        if got is None:
            continue
        np.testing.assert_array_equal(got.cpu().numpy(), getattr(c, name), err_msg=name)


CASES = [
    ("paged_t8", dict(batch=3, seq_lens=[3000, 129, 2056], q_tokens=8, paged=True, seed=81)),
    ("contig_t1", dict(batch=2, seq_lens=[4096, 700], q_tokens=1, paged=False, seed=82)),
    ("fp8idx_t3", dict(batch=2, seq_lens=[2500, 300], q_tokens=3, paged=True, seed=83, idx_fp8=True)),
]


@pytest.mark.parametrize("name,kw", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("scale", [1.0, 1e-3, 40.0])
def test_insert_matches_oracle_bytes(name, kw, scale):
    w = synth.make_workload(name, device="cuda", **kw)
    k, v, ix = _inputs(w, 90 + int(scale * 7) % 13, scale)
    c = _oracle_insert(w, k, v, ix)
    assert _gpu_insert(w, k, v, ix) == (msa.MSA_OK, 0)
    _same(w, c)


def test_insert_ties_zero_and_saturating_rows():
    w = synth.make_workload("ins_edges", 1, [640], 4, paged=True, seed=84, device="cuda")
    w = synth.Workload(**{**w.__dict__, "s_k": 1.0, "s_v": 1.0, "s_idx": 1.0})
    k = torch.zeros(1, 4, 4, 128)
    # block 0 of every K row: amax 6 (scale 1.0) and the E2M1 midpoints
    mids = torch.tensor([6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75,
                         -2.5, -3.5, -5.0, -6.0])
    k[..., :16] = mids
    k[..., 16:32] = 1e30                        # saturating scale and codes
    k[..., 32:48] = -1e-30                      # tiny: scale 0 -> codes 0
    v = torch.randn(1, 4, 4, 128) * 3
    v[0, 1] = 0.0                               # an all-zero token
    ix = torch.randn(1, 4, 128)
    k, v, ix = (x.to(torch.bfloat16).cuda() for x in (k, v, ix))
    c = _oracle_insert(w, k, v, ix)
    assert _gpu_insert(w, k, v, ix) == (msa.MSA_OK, 0)
    _same(w, c)


def test_insert_bad_page_is_reported_and_skipped():
    w = synth.make_workload("ins_bad", 2, [300, 500], 1, paged=True, seed=85, device="cuda")
    pt = w.page_table.clone()
    pt[1, 3] = w.num_pages + 5                  # block of position 499
    wb = synth.Workload(**{**w.__dict__, "page_table": pt})
    k, v, ix = _inputs(w, 86)
    before = w.k_data.clone()
    st, detail = _gpu_insert(wb, k, v, ix)
    assert st == msa.MSA_ERR_DEVICE_BOUNDS and detail == w.num_pages + 5
    # sequence 0's row was written, nothing else changed
    changed = (w.k_data != before).any(dim=(1, 2, 3)).nonzero().flatten().tolist()
    assert changed == [int(w.page_table[0, 299 // 128])]
