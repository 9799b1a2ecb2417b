"""CPU-only checks of the C ABI boundary: the library loads without a GPU,
exports every entry point the header declares, and its host-side argument
checks reject bad calls before any launch (no compute call is made here)."""
import ctypes
import os
import re

import pytest
import torch

import block_sparse_attention_decode_b200 as msa
from block_sparse_attention_decode_b200 import build as msa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    msa_build.build()
    return msa.load()


def header_symbols():
    src = open(os.path.join(ROOT, "include", "msa.h")).read()
    return sorted(set(re.findall(r"MSA_API\s+[\w\s\*]+?\b(msa_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    syms = header_symbols()
    assert len(syms) >= 9
    for s in syms:
        assert hasattr(lib, s), s
    assert sorted(msa.EXPORTED) == syms


def test_status_strings(lib):
    for code in range(7):
        assert msa.status_string(code) and msa.status_string(code) != "unknown status"
    assert msa.status_string(99) == "unknown status"


FAKE = 1 << 20   # an aligned, never-dereferenced address


def _seqs(batch=2, T=1, max_pages=8, lens_ptr=FAKE, pt=None):
    return msa.msa_seqs(page_table=pt, seq_lens=lens_ptr, batch=batch, q_tokens=T, max_pages=max_pages)


def _cache(**kw):
    c = dict(idx_data=FAKE, idx_scale=FAKE, k_data=FAKE, k_scale=FAKE, v_data=FAKE, v_scale=FAKE,
             s_idx=1.0, s_k=1.0, s_v=1.0, num_pages=16, idx_dtype=msa.MSA_IDX_NVFP4)
    c.update(kw)
    return msa.msa_cache(**c)


def test_workspace_size_layout(lib):
    s = _seqs(batch=3, T=2, max_pages=10)
    n = lib.msa_workspace_size(ctypes.byref(s))
    rows = 3 * 2 * 4
    al = lambda x: (x + 255) // 256 * 256
    base = al(8) + al(rows * 10 * 4) + al(rows * 16 * 4) + al(rows * 4)
    assert n >= base and (n - base) % 256 == 0
    for bad in (_seqs(batch=0), _seqs(T=0), _seqs(max_pages=0), _seqs(lens_ptr=None),
                _seqs(lens_ptr=FAKE + 4), _seqs(batch=5000), _seqs(T=2000, max_pages=1)):
        assert lib.msa_workspace_size(ctypes.byref(bad)) == 0


def test_workspace_size_adds_the_decode_once_rows(lib):
    # T x 16 >= 4 x max_pages (every block of a group selected several times
    # over, as in prefill): the size holds 32 KB of E4M3 K and V rows per
    # (sequence, block, KV head); a decode-shaped batch does not
    al = lambda x: (x + 255) // 256 * 256
    dkv = 2 * 71 * 4 * 2 * 128 * 128
    n_pre = lib.msa_workspace_size(ctypes.byref(_seqs(batch=2, T=64, max_pages=71)))
    rows = 2 * 64 * 4
    base = al(8) + al(rows * 71 * 4) + al(rows * 16 * 4) + al(rows * 4)
    assert n_pre >= base + dkv
    n_dec = lib.msa_workspace_size(ctypes.byref(_seqs(batch=2, T=8, max_pages=1024)))
    rows = 2 * 8 * 4
    assert n_dec < al(8) + al(rows * 1024 * 4) + al(rows * 16 * 4) + al(rows * 4) + 2 * 1024 * 4 * 2 * 128 * 128


def _decode(lib, cache, seqs, ws=FAKE, ws_bytes=1 << 40, s_qi=1.0, s_q=1.0, scale=0.1,
            qi=FAKE, q=FAKE, out=FAKE, sel=None):
    return lib.msa_decode(ctypes.byref(cache) if cache is not None else None,
                          ctypes.byref(seqs) if seqs is not None else None, qi, s_qi, q, s_q,
                          scale, out, sel, ws, ws_bytes, None)


@pytest.mark.parametrize("case", [
    "null_cache", "null_seqs", "misaligned_k", "null_idx_scale_nvfp4", "null_idx_scale_exact",
    "misaligned_idx_scale_exact", "bad_dtype", "zero_pages",
    "neg_scale", "nan_scale", "inf_softmax", "misaligned_q", "null_out", "misaligned_sel",
])
def test_host_checks_reject(lib, case):
    cache, seqs = _cache(), _seqs()
    kw = {}
    if case == "null_cache": cache = None
    if case == "null_seqs": seqs = None
    if case == "misaligned_k": cache = _cache(k_data=FAKE + 8)
    if case == "null_idx_scale_nvfp4": cache = _cache(idx_scale=None)
    if case == "null_idx_scale_exact":
        cache = _cache(idx_scale=None, idx_dtype=msa.MSA_IDX_NVFP4_EXACT)
    if case == "misaligned_idx_scale_exact":
        cache = _cache(idx_scale=FAKE + 8, idx_dtype=msa.MSA_IDX_NVFP4_EXACT)
    if case == "bad_dtype": cache = _cache(idx_dtype=7)
    if case == "zero_pages": cache = _cache(num_pages=0)
    if case == "neg_scale": cache = _cache(s_v=-1.0)
    if case == "nan_scale": kw["s_q"] = float("nan")
    if case == "inf_softmax": kw["scale"] = float("inf")
    if case == "misaligned_q": kw["q"] = FAKE + 1
    if case == "null_out": kw["out"] = None
    if case == "misaligned_sel": kw["sel"] = FAKE + 4
    assert _decode(lib, cache, seqs, **kw) == msa.MSA_ERR_INVALID_ARG


def test_workspace_checks(lib):
    cache, seqs = _cache(), _seqs()
    assert _decode(lib, cache, seqs, ws=None) == msa.MSA_ERR_WORKSPACE
    assert _decode(lib, cache, seqs, ws_bytes=100) == msa.MSA_ERR_WORKSPACE
    assert _decode(lib, cache, seqs, ws=FAKE + 8) == msa.MSA_ERR_WORKSPACE
    assert lib.msa_workspace_init(None, 0, None) == msa.MSA_ERR_WORKSPACE


def test_stage_entry_points_check_args(lib):
    cache, seqs = _cache(), _seqs()
    r = lib.msa_indexer_score(ctypes.byref(cache), ctypes.byref(seqs), FAKE, 0.0, None, FAKE,
                              FAKE, 1 << 40, None)
    assert r == msa.MSA_ERR_INVALID_ARG           # s_qi must be > 0
    r = lib.msa_block_maxpool_topk(FAKE, 2, ctypes.byref(seqs), FAKE, FAKE, 1 << 40, None)
    assert r == msa.MSA_ERR_INVALID_ARG           # is_token_level must be 0 or 1
    r = lib.msa_sparse_attn_decode(ctypes.byref(cache), ctypes.byref(seqs), FAKE, 1.0, None,
                                   0.1, FAKE, FAKE, 1 << 40, None)
    assert r == msa.MSA_ERR_INVALID_ARG           # sel required
    assert lib.msa_debug_nvfp4_table(None, None) == msa.MSA_ERR_INVALID_ARG
    for part, nparts in ((0, 0), (1, 1), (-1, 2), (0, 65)):     # context parts out of range
        r = lib.msa_indexer_score_part(ctypes.byref(cache), ctypes.byref(seqs), FAKE, 1.0, None,
                                       FAKE, part, nparts, FAKE, 1 << 40, None)
        assert r == msa.MSA_ERR_INVALID_ARG, (part, nparts)
    fp8 = _cache(idx_scale=None, idx_dtype=msa.MSA_IDX_FP8, s_idx=-2.0)
    r = lib.msa_indexer_score(ctypes.byref(fp8), ctypes.byref(seqs), FAKE, 1.0, None, FAKE,
                              FAKE, 1 << 40, None)
    assert r == msa.MSA_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(msa, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(msa, "_lib", None)
    with pytest.raises(ImportError):
        msa.load()


def test_kv_insert_host_checks(lib):
    s = _seqs()
    c = _cache()
    ws = FAKE
    # null inputs, then a workspace that is too small: rejected before any launch
    st = lib.msa_kv_insert(ctypes.byref(c), ctypes.byref(s), None, ctypes.c_void_p(FAKE),
                           ctypes.c_void_p(FAKE), ctypes.c_void_p(ws), 1 << 30, None)
    assert st == msa.MSA_ERR_INVALID_ARG
    st = lib.msa_kv_insert(ctypes.byref(c), ctypes.byref(s), ctypes.c_void_p(FAKE + 8),
                           ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), ctypes.c_void_p(ws), 1 << 30, None)
    assert st == msa.MSA_ERR_INVALID_ARG     # misaligned
    st = lib.msa_kv_insert(ctypes.byref(c), ctypes.byref(s), ctypes.c_void_p(FAKE),
                           ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), ctypes.c_void_p(ws), 16, None)
    assert st == msa.MSA_ERR_WORKSPACE


def test_binding_refuses_host_tensors(lib):
    t = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(ValueError):
        msa.Cache(t, t, t, t, t, t, 1.0, 1.0, 1.0)
    with pytest.raises(ValueError):
        msa.Seqs(torch.zeros(2, dtype=torch.int32), 1, 4)
