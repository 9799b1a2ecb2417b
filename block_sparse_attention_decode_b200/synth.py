"""Seeded synthetic inputs for the MSA decode path.

This module only *produces input bytes*: pre-quantisation values drawn from
N(0, 1) and encoded into the cache formats the library reads.  It contains
none of the method's arithmetic (no decode, no scoring, no selection, no
attention) and is shared by the CUDA path's tests/benchmark and by the CPU
oracle's tests, which both consume the same bytes.

Encoding used here (an input recipe, not part of the method under test):
  * NVFP4 tensors: blocks of 16 contiguous elements; per-tensor fp32 scale
    ``s_t = amax_nominal / 448`` so that every E2M1 code times its E4M3 block
    scale stays within the E4M3 range; block scale = E4M3(amax16 / (6 s_t))
    by torch's float8 cast; codes = nearest E2M1 magnitude of x/(scale s_t)
    with the sign in bit 3; element 2i in the low nibble of byte i.
  * FP8 tensors (queries, FP8 index keys): E4M3 by torch's float8 cast of
    x / s with a per-tensor scale s.
Every tensor gets its own ``torch.Generator`` stream derived from the
workload seed, so a tensor's bytes do not depend on the order of generation.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

BLOCK = 128
D = 128
G = 4
HPG = 16
HQ = G * HPG
TOPK = 16

# E2M1 magnitudes and the midpoints between neighbours (OCP MX v1.0 table).
_E2M1_MAG = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)
_E2M1_MID = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)

AMAX_NOMINAL = 6.0          # N(0,1) values beyond 6 sigma are clipped by the encoder
S_NVFP4 = AMAX_NOMINAL / 448.0
S_Q = 1.0 / 64.0            # FP8 query scale: N(0,1)/S_Q stays below 448 up to 7 sigma


def _gen(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000003 + int(stream) * 7919 + 17)
    return g


def encode_fp8(x: torch.Tensor, s: float) -> torch.Tensor:
    """x / s rounded to E4M3 by torch's float8 cast, returned as raw bytes."""
    y = (x.float() / s).clamp(-448.0, 448.0)
    return y.to(torch.float8_e4m3fn).view(torch.uint8)


def encode_nvfp4(x: torch.Tensor, s_t: float, scale_floor_byte: int = 0):
    """Encode x [..., 128] into (codes [..., 64] uint8, scales [..., 8] uint8).

    ``scale_floor_byte`` > 0 forces every block-scale byte up to at least that
    value (used by edge-case inputs to exercise the E4M3 saturation of the
    re-rounded products)."""
    assert x.shape[-1] == D
    xf = x.float()
    blk = xf.reshape(*xf.shape[:-1], D // 16, 16)
    amax = blk.abs().amax(dim=-1)
    scale_f = (amax / (6.0 * s_t)).clamp(max=448.0 / 6.0)
    scale_b = scale_f.to(torch.float8_e4m3fn).view(torch.uint8)
    if scale_floor_byte:
        scale_b = torch.maximum(scale_b, torch.full_like(scale_b, scale_floor_byte))
        scale_b = torch.minimum(scale_b, torch.full_like(scale_b, 0x7E))
    scale_dec = scale_b.view(torch.float8_e4m3fn).float()
    denom = (scale_dec * s_t).unsqueeze(-1)
    y = torch.where(denom > 0, blk / torch.where(denom > 0, denom, torch.ones_like(denom)),
                    torch.zeros_like(blk))
    mids = torch.tensor(_E2M1_MID, device=x.device, dtype=torch.float32)
    mag_code = torch.bucketize(y.abs().contiguous(), mids).to(torch.uint8)  # 0..7
    code = mag_code | ((y < 0).to(torch.uint8) << 3)
    code = code.reshape(*xf.shape[:-1], D)
    packed = code[..., 0::2] | (code[..., 1::2] << 4)
    return packed.contiguous(), scale_b.contiguous()


@dataclass
class Workload:
    """One layer's cache plus one step's queries, all as raw bytes (torch)."""
    name: str
    batch: int
    q_tokens: int
    seq_lens: torch.Tensor          # int32 [B]
    max_pages: int
    page_table: torch.Tensor | None  # int32 [B][max_pages] (-1 = unused) or None
    num_pages: int
    idx_fp8: bool
    idx_data: torch.Tensor          # uint8 [P][128][64] or [P][128][128]
    idx_scale: torch.Tensor | None  # uint8 [P][128][8] or None
    k_data: torch.Tensor            # uint8 [P][4][128][64]
    k_scale: torch.Tensor           # uint8 [P][4][128][8]
    v_data: torch.Tensor
    v_scale: torch.Tensor
    qi: torch.Tensor                # uint8 [B][T][4][128] E4M3
    q: torch.Tensor                 # uint8 [B][T][64][128] E4M3
    s_idx: float = S_NVFP4
    s_k: float = S_NVFP4
    s_v: float = S_NVFP4
    s_qi: float = S_Q
    s_q: float = S_Q
    softmax_scale: float = D ** -0.5
    idx_exact: bool = False         # score NVFP4 index keys exactly (no E4M3 re-rounding)
    meta: dict = field(default_factory=dict)

    @property
    def device(self):
        return self.k_data.device


def _page_map(batch, nblk, max_pages, paged, seed, device, prefix_groups=None):
    """Logical (b, i) -> physical page.  Contiguous: page = b*max_pages + i.

    prefix_groups: [(users, prefix_blocks), ...] covering the batch in order:
    the sequences of a group map their first prefix_blocks logical blocks to
    the same physical pages (those of the group's first sequence)."""
    if not paged:
        assert not prefix_groups, "shared prefixes need a page table"
        return None, batch * max_pages
    groups = prefix_groups or [(1, 0)] * batch
    assert sum(u for u, _ in groups) == batch
    total = 0
    b = 0
    for users, pre in groups:
        assert all(pre <= nblk[b + j] for j in range(users))
        total += pre + sum(nblk[b + j] - pre for j in range(users))
        b += users
    perm = torch.randperm(total, generator=_gen(seed, 1, "cpu"))
    pt = torch.full((batch, max_pages), -1, dtype=torch.int32)
    off = 0
    b = 0
    for users, pre in groups:
        shared = perm[off: off + pre].to(torch.int32)
        off += pre
        for j in range(users):
            pt[b, :pre] = shared
            n = nblk[b] - pre
            pt[b, pre: nblk[b]] = perm[off: off + n].to(torch.int32)
            off += n
            b += 1
    return pt.to(device), total


def make_workload(name: str, batch: int, seq_lens, q_tokens: int, *, paged: bool,
                  seed: int, device="cpu", idx_fp8: bool = False, max_pages: int | None = None,
                  plant_every: int = 0, scale_floor_byte: int = 0,
                  neg_scale_frac: float = 0.0, chunk_pages: int = 2048,
                  idx_exact: bool = False, prefix_groups=None) -> Workload:
    """Build a workload.  seq_lens counts the q_tokens new tokens (which are the
    last q_tokens positions of each sequence).

    ``neg_scale_frac`` > 0 sets the sign bit of that fraction of the block-scale
    bytes (index, K and V), to exercise signed E4M3 block scales.

    ``prefix_groups`` = [(users, prefix_blocks), ...] (paged only): consecutive
    groups of sequences whose first prefix_blocks logical blocks are the same
    physical pages, as a serving engine's prefix cache shares them."""
    seq_lens = [int(L) for L in seq_lens]
    assert len(seq_lens) == batch and all(L >= q_tokens >= 1 for L in seq_lens)
    nblk = [(L + BLOCK - 1) // BLOCK for L in seq_lens]
    if max_pages is None:
        max_pages = max(nblk)
    assert max_pages >= max(nblk)
    page_table, num_pages = _page_map(batch, nblk, max_pages, paged, seed, device, prefix_groups)

    # queries (pre-quantisation N(0,1), one stream per tensor)
    qi_f = torch.randn(batch, q_tokens, G, D, generator=_gen(seed, 2, device), device=device)
    q_f = torch.randn(batch, q_tokens, HQ, D, generator=_gen(seed, 3, device), device=device)

    # physical page -> (b, i) for planting and for chunked generation
    if page_table is None:
        owner_b = torch.arange(num_pages, device=device) // max_pages
        owner_i = torch.arange(num_pages, device=device) % max_pages
    else:
        owner_b = torch.empty(num_pages, dtype=torch.long)
        owner_i = torch.empty(num_pages, dtype=torch.long)
        ptc = page_table.cpu()
        for b in range(batch):
            ids = ptc[b, : nblk[b]].long()
            owner_b[ids] = b
            owner_i[ids] = torch.arange(nblk[b])
        owner_b, owner_i = owner_b.to(device), owner_i.to(device)

    idx_row = D if idx_fp8 else D // 2
    idx_data = torch.empty(num_pages, BLOCK, idx_row, dtype=torch.uint8, device=device)
    idx_scale = None if idx_fp8 else torch.empty(num_pages, BLOCK, D // 16, dtype=torch.uint8,
                                                 device=device)
    k_data = torch.empty(num_pages, G, BLOCK, D // 2, dtype=torch.uint8, device=device)
    k_scale = torch.empty(num_pages, G, BLOCK, D // 16, dtype=torch.uint8, device=device)
    v_data = torch.empty_like(k_data)
    v_scale = torch.empty_like(k_scale)

    # planted blocks: +3 sigma along one group's index-query direction
    plant_g = None
    if plant_every:
        gp = _gen(seed, 4, "cpu")
        planted = torch.rand(num_pages, generator=gp) < (1.0 / plant_every)
        which_g = torch.randint(0, G, (num_pages,), generator=gp)
        plant_g = torch.where(planted, which_g, torch.full_like(which_g, -1)).to(device)
        qhat = qi_f[:, 0] / qi_f[:, 0].norm(dim=-1, keepdim=True)   # [B][4][128]

    gi, gk, gv = _gen(seed, 5, device), _gen(seed, 6, device), _gen(seed, 7, device)
    for p0 in range(0, num_pages, chunk_pages):
        p1 = min(num_pages, p0 + chunk_pages)
        n = p1 - p0
        xi = torch.randn(n, BLOCK, D, generator=gi, device=device)
        if plant_g is not None:
            pg = plant_g[p0:p1]
            sel = pg >= 0
            if bool(sel.any()):
                bsel = owner_b[p0:p1][sel]
                gsel = pg[sel]
                xi[sel] += 3.0 * qhat[bsel, gsel].unsqueeze(1)
        if idx_fp8:
            idx_data[p0:p1] = encode_fp8(xi, S_Q)
        else:
            c, s = encode_nvfp4(xi, S_NVFP4, scale_floor_byte)
            idx_data[p0:p1], idx_scale[p0:p1] = c, s
        del xi
        xk = torch.randn(n, G, BLOCK, D, generator=gk, device=device)
        k_data[p0:p1], k_scale[p0:p1] = encode_nvfp4(xk, S_NVFP4, scale_floor_byte)
        del xk
        xv = torch.randn(n, G, BLOCK, D, generator=gv, device=device)
        v_data[p0:p1], v_scale[p0:p1] = encode_nvfp4(xv, S_NVFP4, scale_floor_byte)
        del xv

    if neg_scale_frac > 0:
        gn = _gen(seed, 8, device)
        for t in (idx_scale, k_scale, v_scale):
            if t is None:
                continue
            flip = torch.rand(t.shape, generator=gn, device=device) < neg_scale_frac
            t |= flip.to(torch.uint8) << 7

    if idx_exact and idx_fp8:
        raise ValueError("idx_exact applies to NVFP4 index keys")
    s_idx = S_Q if idx_fp8 else S_NVFP4
    return Workload(
        name=name, batch=batch, q_tokens=q_tokens,
        seq_lens=torch.tensor(seq_lens, dtype=torch.int32, device=device),
        max_pages=max_pages, page_table=page_table, num_pages=num_pages, idx_fp8=idx_fp8,
        idx_data=idx_data, idx_scale=idx_scale, k_data=k_data, k_scale=k_scale,
        v_data=v_data, v_scale=v_scale,
        qi=encode_fp8(qi_f, S_Q), q=encode_fp8(q_f, S_Q),
        s_idx=s_idx, idx_exact=idx_exact, meta={"seed": seed, "paged": paged, "plant_every": plant_every,
                           "scale_floor_byte": scale_floor_byte,
                           "neg_scale_frac": neg_scale_frac},
    )


# ------------------------------------------------------------- workloads --
def ragged_lengths(batch: int, lo: int, hi: int, seed: int):
    """Ragged context lengths: the first sequence is exactly 16 full blocks
    (selection = dense attention), the second has the forced latest block
    holding a single key, the rest are uniform in [lo, hi] with a partially
    filled last block."""
    g = _gen(seed, 8, "cpu")
    out = [lo, lo + 1]
    while len(out) < batch:
        L = int(torch.randint(lo, hi + 1, (1,), generator=g).item())
        if L % BLOCK:
            out.append(L)
    return out[:batch]


WORKLOADS = {
    # name: (kwargs for make_workload, description)
    "ctx4k_b1_t1": dict(batch=1, seq_lens=[4096], q_tokens=1, paged=False, seed=1001),
    "ctx32k_b32_t1": dict(batch=32, seq_lens=[32768] * 32, q_tokens=1, paged=False, seed=1002,
                          plant_every=64),
    "ctx32k_b32_t1_fp8idx": dict(batch=32, seq_lens=[32768] * 32, q_tokens=1, paged=False,
                                 seed=1002, plant_every=64, idx_fp8=True),
    "ctx128k_b64_t8": dict(batch=64, seq_lens=[131072] * 64, q_tokens=8, paged=True, seed=1003),
    "ragged_b16_t1": dict(batch=16, seq_lens=None, q_tokens=1, paged=True, seed=1004),
    "prefill_67584_t2048": dict(batch=1, seq_lens=[65536 + 2048], q_tokens=2048, paged=True,
                                seed=1005),
    # a reduced prefill chunk (256 new tokens), small enough for counter captures
    "prefill_65792_t256": dict(batch=1, seq_lens=[65536 + 256], q_tokens=256, paged=True,
                               seed=1007),
}


def workload(name: str, device="cpu") -> Workload:
    kw = dict(WORKLOADS[name])
    if kw["seq_lens"] is None:
        kw["seq_lens"] = ragged_lengths(kw["batch"], 2048, 262144, kw["seed"])
    return make_workload(name, device=device, **kw)
