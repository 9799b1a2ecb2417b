"""Helpers for the GPU-vs-oracle parity tests.

Tolerances are the stated requirements of the path (written here, used by
every parity test):
  * indexer scores: 1e-3 relative, with the denominator floored at 1e-2 of the
    row's largest |score| so near-zero scores are not judged by a meaningless
    ratio;
  * selected block ids: exact, except blocks whose oracle score lies within
    1e-3 relative of the oracle's boundary (15th-best non-latest) score, where
    either pick is allowed;
  * attention output (bf16): max-abs <= 2e-2 and mean-abs <= 5e-3 against the
    oracle evaluated over the GPU's own selection.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

SCORE_RTOL = 1e-3
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 5e-3


def host_cache(w, seq_ids=None) -> tuple[oracle.Cache, list[int]]:
    """Oracle view of workload w restricted to sequences seq_ids: their pages
    are gathered into a compact host pool behind a new page table."""
    B = w.batch
    seq_ids = list(range(B)) if seq_ids is None else list(seq_ids)
    lens = w.seq_lens.cpu().numpy()
    nblk = [(int(lens[b]) + 127) // 128 for b in seq_ids]
    if w.page_table is None:
        phys = [[b * w.max_pages + i for i in range(n)] for b, n in zip(seq_ids, nblk)]
    else:
        pt = w.page_table.cpu().numpy()
        phys = [[int(pt[b, i]) for i in range(n)] for b, n in zip(seq_ids, nblk)]
    flat = [p for row in phys for p in row]
    idx = torch.tensor(flat, dtype=torch.long, device=w.k_data.device)
    take = lambda t: None if t is None else t.index_select(0, idx).cpu().numpy()
    new_pt = np.full((len(seq_ids), max(nblk)), -1, np.int32)
    off = 0
    for r, n in enumerate(nblk):
        new_pt[r, :n] = np.arange(off, off + n)
        off += n
    c = oracle.Cache(idx_data=take(w.idx_data), idx_scale=take(w.idx_scale),
                     k_data=take(w.k_data), k_scale=take(w.k_scale), v_data=take(w.v_data),
                     v_scale=take(w.v_scale), s_idx=w.s_idx, s_k=w.s_k, s_v=w.s_v,
                     page_table=new_pt, max_pages=max(nblk),
                     seq_lens=np.ascontiguousarray(lens[seq_ids], dtype=np.int32),
                     q_tokens=w.q_tokens, idx_exact=w.idx_exact)
    return c, seq_ids


def host_queries(w, seq_ids):
    qi = w.qi[seq_ids].cpu().numpy()
    q = w.q[seq_ids].cpu().numpy()
    return np.ascontiguousarray(qi), np.ascontiguousarray(q)


def check_scores(gpu: np.ndarray, ref: np.ndarray, what: str):
    """gpu, ref: [..., n] with -inf where no key is visible (must agree)."""
    gi, ri = np.isneginf(gpu), np.isneginf(ref)
    assert np.array_equal(gi, ri), "%s: -inf pattern differs" % what
    fin = ~ri
    g, r = np.where(fin, gpu, 0.0), np.where(fin, ref, 0.0)
    rowmax = np.abs(r).max(axis=-1, keepdims=True)
    denom = np.maximum(np.abs(r), 1e-2 * np.maximum(rowmax, 1e-30))
    rel = np.abs(g - r) / denom
    worst = float(rel.max()) if rel.size else 0.0
    assert worst <= SCORE_RTOL, "%s: max relative error %.3g > %g" % (what, worst, SCORE_RTOL)
    return worst


def check_selection(gpu_sel: np.ndarray, ref_sel: np.ndarray, ref_bscores: np.ndarray,
                    nvis: np.ndarray, what: str) -> int:
    """gpu_sel, ref_sel: [rows][4][16]; ref_bscores [rows][4][max_pages] (f64);
    nvis [rows] visible blocks.  Returns how many rows took a near-tie swap."""
    swaps = 0
    for r in range(gpu_sel.shape[0]):
        nb = int(nvis[r])
        for g in range(4):
            gs = [int(x) for x in gpu_sel[r, g] if x >= 0]
            rs = [int(x) for x in ref_sel[r, g] if x >= 0]
            assert gs == sorted(gs) and len(set(gs)) == len(gs), (what, r, g, gs)
            assert all(x == -1 for x in gpu_sel[r, g, len(gs):]), (what, r, g)
            assert len(gs) == min(nb, 16) and (nb - 1) in gs, (what, r, g, gs, nb)
            if gs == rs:
                continue
            S = ref_bscores[r, g, : nb - 1]
            order = np.lexsort((np.arange(nb - 1), -S))
            boundary = S[order[14]]
            tol = SCORE_RTOL * max(abs(boundary), 1e-2 * np.abs(S).max())
            for blk in set(gs) ^ set(rs):
                assert abs(S[blk] - boundary) <= tol, (
                    "%s: row %d group %d picks %s vs oracle %s (block %d score %.6g, boundary %.6g)"
                    % (what, r, g, gs, rs, blk, S[blk], boundary))
            swaps += 1
    return swaps


def check_output(gpu_bf16: torch.Tensor, ref: np.ndarray, what: str):
    g = gpu_bf16.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= OUT_MAX_ABS, "%s: max-abs %.4g > %g" % (what, mx, OUT_MAX_ABS)
    assert mean <= OUT_MEAN_ABS, "%s: mean-abs %.4g > %g" % (what, mean, OUT_MEAN_ABS)
    return mx, mean
