"""Python binding of libmsa (the MSA decode path on B200, sm_100a).

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libmsa.so``; PyTorch supplies device memory and streams.  The functions
carry the names of the C ABI in ``include/msa.h`` and take torch tensors.
There is no fallback: if the library is missing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa.so")

MSA_OK, MSA_ERR_INVALID_ARG, MSA_ERR_UNSUPPORTED, MSA_ERR_CUDA = 0, 1, 2, 3
MSA_ERR_DEVICE_BOUNDS, MSA_ERR_TIMEOUT, MSA_ERR_WORKSPACE = 4, 5, 6
MSA_IDX_NVFP4, MSA_IDX_FP8, MSA_IDX_NVFP4_EXACT = 0, 1, 2
BLOCK, TOPK, HEAD_DIM, KV_HEADS, Q_HEADS = 128, 16, 128, 4, 64

EXPORTED = [
    "msa_workspace_size", "msa_workspace_init", "msa_indexer_score", "msa_block_maxpool_topk",
    "msa_sparse_attn_decode", "msa_decode", "msa_get_last_error", "msa_debug_nvfp4_table",
    "msa_status_string", "msa_decode_static", "msa_kv_insert", "msa_indexer_score_part",
    "msa_indexer_score_grouped", "msa_decode_grouped",
]
MAX_PARTS = 64
STATIC_WORKSPACE_BYTES = 16 << 20


class MsaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (what, status_string(status), status))


class msa_cache(ctypes.Structure):
    _fields_ = [
        ("idx_data", ctypes.c_void_p), ("idx_scale", ctypes.c_void_p),
        ("k_data", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
        ("v_data", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
        ("s_idx", ctypes.c_float), ("s_k", ctypes.c_float), ("s_v", ctypes.c_float),
        ("num_pages", ctypes.c_int32), ("idx_dtype", ctypes.c_int32),
    ]


class msa_seqs(ctypes.Structure):
    _fields_ = [
        ("page_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
        ("batch", ctypes.c_int32), ("q_tokens", ctypes.c_int32), ("max_pages", ctypes.c_int32),
    ]


class msa_prefix_groups(ctypes.Structure):
    _fields_ = [
        ("seq_start", ctypes.c_void_p), ("prefix_blocks", ctypes.c_void_p),
        ("num_groups", ctypes.c_int32),
    ]


_lib = None


def load() -> ctypes.CDLL:
    """Load libmsa.so (built in-tree by ``build.py``); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("libmsa.so not built: run `python -m block_sparse_attention_decode_b200.build`"
                          " (there is no fallback path)")
    L = ctypes.CDLL(LIB_PATH)
    P, vp, f32, i32, sz = ctypes.POINTER, ctypes.c_void_p, ctypes.c_float, ctypes.c_int32, ctypes.c_size_t
    L.msa_workspace_size.restype = sz
    L.msa_workspace_size.argtypes = [P(msa_seqs)]
    L.msa_workspace_init.restype = ctypes.c_int
    L.msa_workspace_init.argtypes = [vp, sz, vp]
    L.msa_indexer_score.restype = ctypes.c_int
    L.msa_indexer_score.argtypes = [P(msa_cache), P(msa_seqs), vp, f32, vp, vp, vp, sz, vp]
    L.msa_indexer_score_part.restype = ctypes.c_int
    L.msa_indexer_score_part.argtypes = [P(msa_cache), P(msa_seqs), vp, f32, vp, vp, i32, i32, vp,
                                         sz, vp]
    L.msa_block_maxpool_topk.restype = ctypes.c_int
    L.msa_block_maxpool_topk.argtypes = [vp, i32, P(msa_seqs), vp, vp, sz, vp]
    L.msa_indexer_score_grouped.restype = ctypes.c_int
    L.msa_indexer_score_grouped.argtypes = [P(msa_cache), P(msa_seqs), P(msa_prefix_groups), vp, f32,
                                            vp, vp, vp, sz, vp]
    L.msa_decode_grouped.restype = ctypes.c_int
    L.msa_decode_grouped.argtypes = [P(msa_cache), P(msa_seqs), P(msa_prefix_groups), vp, f32, vp,
                                     f32, f32, vp, vp, vp, sz, vp]
    L.msa_sparse_attn_decode.restype = ctypes.c_int
    L.msa_sparse_attn_decode.argtypes = [P(msa_cache), P(msa_seqs), vp, f32, vp, f32, vp, vp, sz, vp]
    L.msa_decode.restype = ctypes.c_int
    L.msa_decode.argtypes = [P(msa_cache), P(msa_seqs), vp, f32, vp, f32, f32, vp, vp, vp, sz, vp]
    L.msa_decode_static.restype = ctypes.c_int
    L.msa_decode_static.argtypes = [P(msa_cache), P(msa_seqs), vp, f32, vp, f32, f32, vp, vp, vp]
    L.msa_kv_insert.restype = ctypes.c_int
    L.msa_kv_insert.argtypes = [P(msa_cache), P(msa_seqs), vp, vp, vp, vp, sz, vp]
    L.msa_get_last_error.restype = ctypes.c_int
    L.msa_get_last_error.argtypes = [vp, vp, P(i32)]
    L.msa_debug_nvfp4_table.restype = ctypes.c_int
    L.msa_debug_nvfp4_table.argtypes = [vp, vp]
    L.msa_status_string.restype = ctypes.c_char_p
    L.msa_status_string.argtypes = [ctypes.c_int]
    _lib = L
    return L


def status_string(status: int) -> str:
    return load().msa_status_string(int(status)).decode()


def _ptr(t):
    if t is not None and not t.is_cuda:
        raise ValueError("libmsa takes CUDA tensors; got a tensor on %s" % t.device)
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def _check(status: int, what: str):
    if status != MSA_OK:
        raise MsaError(status, what)


def _device_tensors(ts):
    """The library takes device pointers only: refuse host tensors here rather
    than hand a kernel an address it cannot read."""
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libmsa takes CUDA tensors; got a tensor on %s" % t.device)


class Cache:
    """Holds the cache tensors (keeps them alive) and their C description."""

    def __init__(self, idx_data, idx_scale, k_data, k_scale, v_data, v_scale,
                 s_idx: float, s_k: float, s_v: float, idx_exact: bool = False):
        """idx_scale None = FP8 index keys; idx_exact = score NVFP4 index keys
        at their exact value (MSA_IDX_NVFP4_EXACT)."""
        self.tensors = (idx_data, idx_scale, k_data, k_scale, v_data, v_scale)
        _device_tensors(self.tensors)
        if idx_scale is None:
            dtype = MSA_IDX_FP8
        else:
            dtype = MSA_IDX_NVFP4_EXACT if idx_exact else MSA_IDX_NVFP4
        self.c = msa_cache(
            idx_data=idx_data.data_ptr(),
            idx_scale=idx_scale.data_ptr() if idx_scale is not None else None,
            k_data=k_data.data_ptr(), k_scale=k_scale.data_ptr(),
            v_data=v_data.data_ptr(), v_scale=v_scale.data_ptr(),
            s_idx=s_idx, s_k=s_k, s_v=s_v, num_pages=int(k_data.shape[0]),
            idx_dtype=dtype)


class Seqs:
    """Holds page table / lengths (device int32) and their C description."""

    def __init__(self, seq_lens, q_tokens: int, max_pages: int, page_table=None):
        self.tensors = (seq_lens, page_table)
        _device_tensors(self.tensors)
        self.c = msa_seqs(page_table=page_table.data_ptr() if page_table is not None else None,
                          seq_lens=seq_lens.data_ptr(), batch=int(seq_lens.shape[0]),
                          q_tokens=int(q_tokens), max_pages=int(max_pages))

    @property
    def rows(self) -> int:
        return self.c.batch * self.c.q_tokens * KV_HEADS


class PrefixGroups:
    """Groups of consecutive sequences sharing a cached prefix (device int32
    tensors seq_start [G+1] and prefix_blocks [G]) and their C description."""

    def __init__(self, seq_start, prefix_blocks):
        self.tensors = (seq_start, prefix_blocks)
        _device_tensors(self.tensors)
        self.c = msa_prefix_groups(seq_start=seq_start.data_ptr(),
                                   prefix_blocks=prefix_blocks.data_ptr(),
                                   num_groups=int(prefix_blocks.shape[0]))

    @classmethod
    def of(cls, groups, device="cuda"):
        """From [(users, prefix_blocks), ...] covering the batch in order."""
        start = [0]
        for users, _ in groups:
            start.append(start[-1] + int(users))
        return cls(torch.tensor(start, dtype=torch.int32, device=device),
                   torch.tensor([int(p) for _, p in groups], dtype=torch.int32, device=device))


def cache_of(w) -> Cache:
    return Cache(w.idx_data, w.idx_scale, w.k_data, w.k_scale, w.v_data, w.v_scale,
                 w.s_idx, w.s_k, w.s_v, idx_exact=w.idx_exact)


def seqs_of(w) -> Seqs:
    return Seqs(w.seq_lens, w.q_tokens, w.max_pages, w.page_table)


# ----------------------------------------------------------- the C ABI ----
def msa_workspace_size(seqs: Seqs) -> int:
    n = load().msa_workspace_size(ctypes.byref(seqs.c))
    if n == 0:
        raise MsaError(MSA_ERR_INVALID_ARG, "msa_workspace_size")
    return int(n)


def msa_workspace_init(ws: torch.Tensor, stream=None):
    _check(load().msa_workspace_init(_ptr(ws), _nbytes(ws), _stream(stream)),
           "msa_workspace_init")


def alloc_workspace(seqs: Seqs, device=None) -> torch.Tensor:
    ws = torch.empty(msa_workspace_size(seqs), dtype=torch.uint8, device=device or "cuda")
    msa_workspace_init(ws)
    return ws


def msa_indexer_score(cache: Cache, seqs: Seqs, qi, s_qi: float, token_scores, block_scores,
                      ws, stream=None):
    """Indexer scores and block max-pool.  qi: uint8 E4M3 [B][T][4][128];
    token_scores: float32 [B][T][4][max_pages*128] or None; block_scores:
    float32 [B][T][4][max_pages]."""
    _check(load().msa_indexer_score(ctypes.byref(cache.c), ctypes.byref(seqs.c), _ptr(qi), s_qi,
                                    _ptr(token_scores), _ptr(block_scores), _ptr(ws),
                                    _nbytes(ws), _stream(stream)), "msa_indexer_score")


def msa_indexer_score_part(cache: Cache, seqs: Seqs, qi, s_qi: float, token_scores, block_scores,
                           part: int, nparts: int, ws, stream=None):
    """msa_indexer_score over part `part` of `nparts` of every sequence's
    blocks only (context parallelism); the other entries are not written."""
    _check(load().msa_indexer_score_part(ctypes.byref(cache.c), ctypes.byref(seqs.c), _ptr(qi),
                                         s_qi, _ptr(token_scores), _ptr(block_scores), int(part),
                                         int(nparts), _ptr(ws), _nbytes(ws), _stream(stream)),
           "msa_indexer_score_part")


def msa_block_maxpool_topk(scores, is_token_level: bool, seqs: Seqs, sel, ws, stream=None):
    """Top-16 blocks per (b, t, g), the latest always kept: sel int32
    [B][T][4][16], ascending, -1 padded.  scores: block scores, or token
    scores (max-pooled first) when is_token_level."""
    _check(load().msa_block_maxpool_topk(_ptr(scores), int(bool(is_token_level)),
                                         ctypes.byref(seqs.c), _ptr(sel), _ptr(ws), _nbytes(ws),
                                         _stream(stream)), "msa_block_maxpool_topk")


def msa_sparse_attn_decode(cache: Cache, seqs: Seqs, q, s_q: float, sel, softmax_scale: float,
                           out, ws, stream=None):
    """Attention over the selected blocks.  q: uint8 E4M3 [B][T][64][128];
    sel: int32 [B][T][4][16]; out: bfloat16 [B][T][64][128]."""
    _check(load().msa_sparse_attn_decode(ctypes.byref(cache.c), ctypes.byref(seqs.c), _ptr(q), s_q,
                                         _ptr(sel), softmax_scale, _ptr(out), _ptr(ws), _nbytes(ws),
                                         _stream(stream)), "msa_sparse_attn_decode")


def msa_decode(cache: Cache, seqs: Seqs, qi, s_qi: float, q, s_q: float, softmax_scale: float,
               out, sel_out, ws, stream=None):
    """The whole decode step (indexer, top-16, attention) on `stream`;
    sel_out (int32 [B][T][4][16]) optional."""
    _check(load().msa_decode(ctypes.byref(cache.c), ctypes.byref(seqs.c), _ptr(qi), s_qi, _ptr(q),
                             s_q, softmax_scale, _ptr(out), _ptr(sel_out), _ptr(ws), _nbytes(ws),
                             _stream(stream)), "msa_decode")


def msa_indexer_score_grouped(cache: Cache, seqs: Seqs, groups: PrefixGroups, qi, s_qi: float,
                              token_scores, block_scores, ws, stream=None):
    """msa_indexer_score with shared-prefix pages decoded once per tile of
    the group's index queries (same scores)."""
    _check(load().msa_indexer_score_grouped(ctypes.byref(cache.c), ctypes.byref(seqs.c),
                                            ctypes.byref(groups.c), _ptr(qi), s_qi,
                                            _ptr(token_scores), _ptr(block_scores), _ptr(ws),
                                            _nbytes(ws), _stream(stream)), "msa_indexer_score_grouped")


def msa_decode_grouped(cache: Cache, seqs: Seqs, groups: PrefixGroups, qi, s_qi: float, q,
                       s_q: float, softmax_scale: float, out, sel_out, ws, stream=None):
    """msa_decode over a batch with shared prefixes (the grouped indexer)."""
    _check(load().msa_decode_grouped(ctypes.byref(cache.c), ctypes.byref(seqs.c),
                                     ctypes.byref(groups.c), _ptr(qi), s_qi, _ptr(q), s_q,
                                     softmax_scale, _ptr(out), _ptr(sel_out), _ptr(ws), _nbytes(ws),
                                     _stream(stream)), "msa_decode_grouped")


def msa_decode_static(cache: Cache, seqs: Seqs, qi, s_qi: float, q, s_q: float,
                      softmax_scale: float, out, sel_out, stream=None):
    """msa_decode with the library's fixed scratch array instead of a workspace
    (for callers that cannot allocate device memory on the calling path)."""
    _check(load().msa_decode_static(ctypes.byref(cache.c), ctypes.byref(seqs.c), _ptr(qi), s_qi,
                                    _ptr(q), s_q, softmax_scale, _ptr(out), _ptr(sel_out),
                                    _stream(stream)), "msa_decode_static")


def msa_kv_insert(cache: Cache, seqs: Seqs, k_new, v_new, idx_new, ws, stream=None):
    """Quantise the new tokens (bf16 tensors [B][T][4][128], [B][T][4][128],
    [B][T][128]) into the cache the descriptor points to."""
    for x in (k_new, v_new, idx_new):
        if x.dtype != torch.bfloat16 or not x.is_contiguous():
            raise ValueError("msa_kv_insert takes contiguous bfloat16 tensors")
    _check(load().msa_kv_insert(ctypes.byref(cache.c), ctypes.byref(seqs.c), _ptr(k_new), _ptr(v_new),
                                _ptr(idx_new), _ptr(ws), _nbytes(ws), _stream(stream)), "msa_kv_insert")


def msa_get_last_error(ws, stream=None):
    """(status, detail) of the first device-side error since the last call;
    synchronises the stream and clears the record."""
    detail = ctypes.c_int32(0)
    st = load().msa_get_last_error(_ptr(ws), _stream(stream), ctypes.byref(detail))
    return int(st), int(detail.value)


def msa_debug_nvfp4_table(out, stream=None):
    _check(load().msa_debug_nvfp4_table(_ptr(out), _stream(stream)), "msa_debug_nvfp4_table")
