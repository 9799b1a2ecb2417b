"""Independent decoding of the cache bytes with torch's own float8 conversions.

Used only to PIN the oracle: the E4M3 decode and the saturating
round-to-nearest-even come from torch's float8_e4m3fn cast (a library
routine), the E2M1 magnitudes from the OCP MX v1.0 table
(``golden/e2m1_values.txt``), and the contractions from torch.matmul /
scaled_dot_product_attention in float64.  Nothing here calls the oracle or
the CUDA library.
"""
from __future__ import annotations

import os

import numpy as np
import torch

_GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def e2m1_table() -> torch.Tensor:
    vals = {}
    for line in open(os.path.join(_GOLDEN, "e2m1_values.txt")):
        line = line.split("#")[0].strip()
        if line:
            c, v = line.split()
            vals[int(c, 0)] = float(v)
    assert sorted(vals) == list(range(16))
    return torch.tensor([vals[c] for c in range(16)], dtype=torch.float64)


def e4m3_to_f64(b: torch.Tensor) -> torch.Tensor:
    return b.to(torch.uint8).contiguous().view(torch.float8_e4m3fn).to(torch.float64)


def round_e4m3_sat(x: torch.Tensor) -> torch.Tensor:
    """Saturating RNE to E4M3 through torch's cast (clamp first: torch's cast
    itself does not saturate)."""
    return x.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).to(torch.float64)


def decode_nvfp4(data: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """data [..., 64] uint8, scale [..., 8] uint8 -> [..., 128] float64 values
    (before the per-tensor scale)."""
    t = e2m1_table()
    lo = (data & 15).long()
    hi = (data >> 4).long()
    codes = torch.stack([lo, hi], dim=-1).reshape(*data.shape[:-1], 128)
    e2 = t[codes]
    sc = e4m3_to_f64(scale).repeat_interleave(16, dim=-1)
    return round_e4m3_sat(e2 * sc)


def logical_rows(page_table, seq_lens, max_pages, b, arr_per_page: torch.Tensor, L=None):
    """Gather a per-page array [P][128][...] into logical token order for
    sequence b: [L][...]."""
    L = int(seq_lens[b]) if L is None else L
    nb = (L + 127) // 128
    if page_table is None:
        pages = [b * max_pages + i for i in range(nb)]
    else:
        pages = [int(page_table[b][i]) for i in range(nb)]
    out = torch.cat([arr_per_page[p] for p in pages], dim=0)
    return out[:L]


def index_keys(w, b) -> torch.Tensor:
    """Decoded index keys of sequence b in token order [L][128], times s_idx."""
    if w.idx_fp8:
        per_page = e4m3_to_f64(w.idx_data)
    else:
        per_page = decode_nvfp4(w.idx_data, w.idx_scale)
    return logical_rows(w.page_table, w.seq_lens, w.max_pages, b, per_page) * w.s_idx


def kv(w, b, which: str) -> torch.Tensor:
    """Decoded K or V of sequence b: [4][L][128], times s_k / s_v."""
    data = w.k_data if which == "k" else w.v_data
    scale = w.k_scale if which == "k" else w.v_scale
    s = w.s_k if which == "k" else w.s_v
    per_page = decode_nvfp4(data, scale).permute(0, 2, 1, 3)  # [P][128][4][128]
    rows = logical_rows(w.page_table, w.seq_lens, w.max_pages, b, per_page)  # [L][4][128]
    return rows.permute(1, 0, 2).contiguous() * s


def token_scores(w, b, t) -> torch.Tensor:
    """[4][pos+1] float64 index scores by torch.matmul."""
    L = int(w.seq_lens[b])
    pos = L - w.q_tokens + t
    K = index_keys(w, b)[: pos + 1]
    qi = e4m3_to_f64(w.qi[b, t]) * w.s_qi  # [4][128]
    return qi @ K.T


def block_scores(w, b, t) -> torch.Tensor:
    """[4][max_pages] by max_pool1d over the token scores (-inf padded)."""
    s = token_scores(w, b, t)
    n = s.shape[1]
    nb = (n + 127) // 128
    pad = torch.full((4, nb * 128 - n), -np.inf, dtype=torch.float64)
    sp = torch.cat([s, pad], dim=1).unsqueeze(0)
    pooled = torch.nn.functional.max_pool1d(sp, kernel_size=128, stride=128)[0]
    out = torch.full((4, w.max_pages), -np.inf, dtype=torch.float64)
    out[:, :nb] = pooled
    return out


def select_by_sort(scores_row: np.ndarray, nb: int) -> list[int]:
    """Top-16 with the latest block forced, by a library sort: numpy lexsort
    on (id asc) within (score desc)."""
    if nb <= 16:
        return list(range(nb))
    cand = np.arange(nb - 1)
    order = np.lexsort((cand, -scores_row[: nb - 1]))
    return sorted([int(i) for i in order[:15]] + [nb - 1])


def attention_sdpa(w, b, t, sel_bt: np.ndarray, softmax_scale: float) -> torch.Tensor:
    """[64][128] float64 by scaled_dot_product_attention with a boolean mask
    built from the selection (keys of selected blocks up to the position)."""
    L = int(w.seq_lens[b])
    pos = L - w.q_tokens + t
    K = kv(w, b, "k")[:, : pos + 1]
    V = kv(w, b, "v")[:, : pos + 1]
    q = e4m3_to_f64(w.q[b, t]) * w.s_q  # [64][128]
    out = torch.empty(64, 128, dtype=torch.float64)
    for g in range(4):
        mask = torch.zeros(pos + 1, dtype=torch.bool)
        for blk in sel_bt[g]:
            if blk >= 0:
                mask[blk * 128: min(pos + 1, blk * 128 + 128)] = True
        qg = q[g * 16:(g + 1) * 16].unsqueeze(0)          # [1][16][128]
        o = torch.nn.functional.scaled_dot_product_attention(
            qg, K[g].unsqueeze(0), V[g].unsqueeze(0), attn_mask=mask.unsqueeze(0).unsqueeze(0),
            scale=softmax_scale)
        out[g * 16:(g + 1) * 16] = o[0]
    return out
