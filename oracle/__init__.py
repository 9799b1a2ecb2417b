"""Float64 CPU oracle of the MSA decode path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it, and this package never imports the
product path: the two share nothing but the seeded input generator.

The arithmetic lives in ``msa_oracle.c`` (plain C, float64, pthreads); this
module compiles it with gcc on first use and wraps it with ctypes.  Every
function works on explicit (sequence, token) *rows* so that a test can ask
for a sampled subset of a large workload.

Method source: the vLLM blog post "vLLM 為 MiniMax-M3.1-Flash 提供 Day-0 支援"
(hot.atechcom.net), sections "MSA primer", "NVIDIA Blackwell optimized MSA
kernels" and "NVIDIA Rubin optimized MSA"; number formats from OCP MX v1.0.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

BLOCK = 128
TOPK = 16
D = 128
G = 4
HPG = 16
HQ = G * HPG


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no GPU involved). Returns the .so path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-shared", "-fPIC",
                               "-pthread", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Cache(ctypes.Structure):
    _fields_ = [
        ("idx_data", ctypes.c_void_p), ("idx_scale", ctypes.c_void_p),
        ("k_data", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
        ("v_data", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
        ("s_idx", ctypes.c_double), ("s_k", ctypes.c_double), ("s_v", ctypes.c_double),
        ("num_pages", ctypes.c_int64), ("idx_mode", ctypes.c_int),
        ("page_table", ctypes.c_void_p), ("max_pages", ctypes.c_int64),
        ("seq_lens", ctypes.c_void_p), ("batch", ctypes.c_int), ("q_tokens", ctypes.c_int),
    ]


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.orc_e2m1.restype = ctypes.c_double
        L.orc_e2m1.argtypes = [ctypes.c_uint]
        L.orc_e4m3.restype = ctypes.c_double
        L.orc_e4m3.argtypes = [ctypes.c_uint]
        L.orc_e4m3_round.restype = ctypes.c_uint
        L.orc_e4m3_round.argtypes = [ctypes.c_double]
        L.orc_nvfp4_elem.restype = ctypes.c_double
        L.orc_nvfp4_elem.argtypes = [ctypes.c_uint, ctypes.c_uint]
        L.orc_decode_nvfp4_row.restype = None
        L.orc_decode_nvfp4_row.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.orc_set_threads.argtypes = [ctypes.c_int]
        L.orc_get_threads.restype = ctypes.c_int
        L.orc_indexer.restype = ctypes.c_int
        L.orc_indexer.argtypes = [ctypes.POINTER(_Cache), ctypes.c_void_p, ctypes.c_double,
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                  ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        L.orc_select.restype = ctypes.c_int
        L.orc_select.argtypes = [ctypes.POINTER(_Cache), ctypes.c_void_p, ctypes.c_void_p,
                                 ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
        L.orc_attention.restype = ctypes.c_int
        L.orc_attention.argtypes = [ctypes.POINTER(_Cache), ctypes.c_void_p, ctypes.c_double,
                                    ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
        L.orc_e2m1_round.restype = ctypes.c_uint
        L.orc_e2m1_round.argtypes = [ctypes.c_double]
        L.orc_nvfp4_encode_row.restype = None
        L.orc_nvfp4_encode_row.argtypes = [ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p,
                                           ctypes.c_void_p]
        L.orc_fp8_encode_row.restype = None
        L.orc_fp8_encode_row.argtypes = [ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p]
        L.orc_kv_insert.restype = ctypes.c_int
        L.orc_kv_insert.argtypes = [ctypes.POINTER(_Cache), ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_float, ctypes.c_float, ctypes.c_float]
        L.orc_set_threads(os.cpu_count() or 1)
        _lib = L
    return _lib


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def get_threads() -> int:
    return int(lib().orc_get_threads())


# ---------------------------------------------------------------- formats --
def e2m1(code: int) -> float:
    return lib().orc_e2m1(code)


def e4m3(byte: int) -> float:
    return lib().orc_e4m3(byte)


def e4m3_round(x: float) -> int:
    return lib().orc_e4m3_round(float(x))


def nvfp4_elem(code: int, scale_byte: int) -> float:
    return lib().orc_nvfp4_elem(code, scale_byte)


def decode_nvfp4_row(data64: np.ndarray, scale8: np.ndarray) -> np.ndarray:
    data64 = np.ascontiguousarray(data64, dtype=np.uint8)
    scale8 = np.ascontiguousarray(scale8, dtype=np.uint8)
    assert data64.size == 64 and scale8.size == 8
    out = np.empty(128, np.float64)
    lib().orc_decode_nvfp4_row(data64.ctypes.data, scale8.ctypes.data, out.ctypes.data)
    return out


def e2m1_round(y: float) -> int:
    """Nearest E2M1 magnitude code (0..7) of y >= 0, ties to the even code."""
    return lib().orc_e2m1_round(float(y))


def nvfp4_encode_row(x: np.ndarray, s_t: float):
    """128 fp32 values -> (codes uint8[64], scales uint8[8]) (the insert reading)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    assert x.size == 128
    data = np.zeros(64, np.uint8)
    sc = np.zeros(8, np.uint8)
    lib().orc_nvfp4_encode_row(x.ctypes.data, float(s_t), data.ctypes.data, sc.ctypes.data)
    return data, sc


def fp8_encode_row(x: np.ndarray, s_t: float) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    assert x.size == 128
    out = np.zeros(128, np.uint8)
    lib().orc_fp8_encode_row(x.ctypes.data, float(s_t), out.ctypes.data)
    return out


# ------------------------------------------------------------------ cache --
@dataclass
class Cache:
    """Host (numpy) view of one layer's paged cache, in the library's layout."""
    idx_data: np.ndarray          # uint8 [P][128][64] (NVFP4) or [P][128][128] (FP8)
    idx_scale: np.ndarray | None  # uint8 [P][128][8] or None for FP8
    k_data: np.ndarray            # uint8 [P][4][128][64]
    k_scale: np.ndarray           # uint8 [P][4][128][8]
    v_data: np.ndarray
    v_scale: np.ndarray
    s_idx: float
    s_k: float
    s_v: float
    page_table: np.ndarray | None  # int32 [B][max_pages] or None (contiguous)
    max_pages: int
    seq_lens: np.ndarray           # int32 [B]
    q_tokens: int
    idx_exact: bool = False        # NVFP4 index keys scored at their exact value (no E4M3 re-rounding)

    def _c(self) -> _Cache:
        arrs = [self.idx_data, self.k_data, self.k_scale, self.v_data, self.v_scale, self.seq_lens]
        for a in arrs:
            assert a.flags.c_contiguous
        c = _Cache()
        c.idx_data = self.idx_data.ctypes.data
        c.idx_scale = self.idx_scale.ctypes.data if self.idx_scale is not None else None
        c.k_data, c.k_scale = self.k_data.ctypes.data, self.k_scale.ctypes.data
        c.v_data, c.v_scale = self.v_data.ctypes.data, self.v_scale.ctypes.data
        c.s_idx, c.s_k, c.s_v = float(self.s_idx), float(self.s_k), float(self.s_v)
        c.num_pages = int(self.k_data.shape[0])
        c.idx_mode = 1 if self.idx_scale is None else (2 if self.idx_exact else 0)
        c.page_table = self.page_table.ctypes.data if self.page_table is not None else None
        c.max_pages = int(self.max_pages)
        c.seq_lens = self.seq_lens.ctypes.data
        c.batch = int(self.seq_lens.shape[0])
        c.q_tokens = int(self.q_tokens)
        return c


def _rows(rows):
    rb = np.ascontiguousarray([r[0] for r in rows], dtype=np.int32)
    rt = np.ascontiguousarray([r[1] for r in rows], dtype=np.int32)
    return rb, rt


def all_rows(cache: Cache):
    return [(b, t) for b in range(cache.seq_lens.shape[0]) for t in range(cache.q_tokens)]


def indexer(cache: Cache, qi: np.ndarray, s_qi: float, rows, token_scores: bool = True,
            ctx_cap: int | None = None):
    """Token scores [n][4][ctx_cap] (NaN where not computed) and block scores
    [n][4][max_pages] (-inf for blocks without a visible key) for the rows."""
    qi = np.ascontiguousarray(qi, dtype=np.uint8)
    rb, rt = _rows(rows)
    n = len(rows)
    cap = int(ctx_cap if ctx_cap is not None else cache.max_pages * BLOCK)
    sc = np.full((n, G, cap), np.nan, np.float64) if token_scores else None
    bs = np.empty((n, G, cache.max_pages), np.float64)
    c = cache._c()
    rc = lib().orc_indexer(ctypes.byref(c), qi.ctypes.data, float(s_qi), rb.ctypes.data,
                           rt.ctypes.data, n, sc.ctypes.data if sc is not None else None, cap,
                           bs.ctypes.data)
    if rc:
        raise ValueError("oracle indexer: bad row or page (status %d)" % rc)
    return sc, bs


def select(cache: Cache, rows, block_scores: np.ndarray) -> np.ndarray:
    """Selected block ids [n][4][16], ascending, -1 padded."""
    block_scores = np.ascontiguousarray(block_scores, dtype=np.float64)
    rb, rt = _rows(rows)
    sel = np.empty((len(rows), G, TOPK), np.int32)
    c = cache._c()
    rc = lib().orc_select(ctypes.byref(c), rb.ctypes.data, rt.ctypes.data, len(rows),
                          block_scores.ctypes.data, sel.ctypes.data)
    if rc:
        raise ValueError("oracle select: bad row")
    return sel


def attention(cache: Cache, q: np.ndarray, s_q: float, softmax_scale: float, rows,
              sel: np.ndarray) -> np.ndarray:
    """Attention output [n][64][128] (float64) over the given selection."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    rb, rt = _rows(rows)
    out = np.empty((len(rows), HQ, D), np.float64)
    c = cache._c()
    rc = lib().orc_attention(ctypes.byref(c), q.ctypes.data, float(s_q), float(softmax_scale),
                             rb.ctypes.data, rt.ctypes.data, len(rows), sel.ctypes.data,
                             out.ctypes.data)
    if rc:
        raise ValueError("oracle attention: bad row or page (status %d)" % rc)
    return out


def decode(cache: Cache, qi, s_qi, q, s_q, softmax_scale, rows):
    """The whole path for the rows: (block_scores, sel, out)."""
    _, bs = indexer(cache, qi, s_qi, rows, token_scores=False)
    sel = select(cache, rows, bs)
    out = attention(cache, q, s_q, softmax_scale, rows, sel)
    return bs, sel, out


def kv_insert(cache: Cache, k_new: np.ndarray, v_new: np.ndarray, idx_new: np.ndarray) -> int:
    """Quantise the T new tokens of every sequence into `cache` in place.
    k_new, v_new: fp32 [B][T][4][128]; idx_new: fp32 [B][T][128]."""
    k_new = np.ascontiguousarray(k_new, dtype=np.float32)
    v_new = np.ascontiguousarray(v_new, dtype=np.float32)
    idx_new = np.ascontiguousarray(idx_new, dtype=np.float32)
    c = cache._c()
    return int(lib().orc_kv_insert(ctypes.byref(c), k_new.ctypes.data, v_new.ctypes.data,
                                   idx_new.ctypes.data, np.float32(cache.s_idx),
                                   np.float32(cache.s_k), np.float32(cache.s_v)))
