"""GPU checks of the C ABI's memory checks and of one process driving two
devices.

The library checks every buffer before any launch: host memory (pinned or
pageable) or a buffer whose last byte is not device memory is an argument
error, returned without a launch, so that a C caller's wrong pointer never
reaches a kernel.  The calls here go straight to the C ABI through ctypes
(the Python binding refuses host tensors before the call).
"""
import ctypes

import pytest
import torch

import block_sparse_attention_decode_b200 as msa
from block_sparse_attention_decode_b200 import build as msa_build
from block_sparse_attention_decode_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    msa_build.build()
    return msa.load()


@pytest.fixture(scope="module")
def wl():
    return synth.make_workload("boundary", 2, [3000, 700], 2, paged=True, seed=61, device="cuda")


def _vp(t):
    return ctypes.c_void_p(t.data_ptr())


def _cache_struct(w, **override):
    f = dict(idx_data=w.idx_data, idx_scale=w.idx_scale, k_data=w.k_data, k_scale=w.k_scale,
             v_data=w.v_data, v_scale=w.v_scale)
    f.update(override)
    return msa.msa_cache(idx_data=f["idx_data"].data_ptr(), idx_scale=f["idx_scale"].data_ptr(),
                         k_data=f["k_data"].data_ptr(), k_scale=f["k_scale"].data_ptr(),
                         v_data=f["v_data"].data_ptr(), v_scale=f["v_scale"].data_ptr(),
                         s_idx=w.s_idx, s_k=w.s_k, s_v=w.s_v, num_pages=int(w.k_data.shape[0]),
                         idx_dtype=msa.MSA_IDX_NVFP4)


def _seqs_struct(w, seq_lens=None):
    lens = w.seq_lens if seq_lens is None else seq_lens
    return msa.msa_seqs(page_table=w.page_table.data_ptr(), seq_lens=lens.data_ptr(),
                        batch=w.batch, q_tokens=w.q_tokens, max_pages=w.max_pages)


def _buffers(w):
    out = torch.zeros(w.batch, w.q_tokens, 64, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.zeros(w.batch, w.q_tokens, 4, 16, dtype=torch.int32, device="cuda")
    ws = msa.alloc_workspace(msa.seqs_of(w))
    return out, sel, ws


def _decode(lib, w, cache, seqs, qi, q, out, sel, ws):
    return lib.msa_decode(ctypes.byref(cache), ctypes.byref(seqs), _vp(qi), w.s_qi, _vp(q), w.s_q,
                          w.softmax_scale, _vp(out), _vp(sel), _vp(ws), ws.numel(), None)


def _flags_clear(ws):
    torch.cuda.synchronize()
    assert msa.msa_get_last_error(ws) == (msa.MSA_OK, 0)


def test_decode_rejects_host_buffers(lib, wl):
    w = wl
    out, sel, ws = _buffers(w)
    cache, seqs = _cache_struct(w), _seqs_struct(w)
    # the valid call first: it runs
    assert _decode(lib, w, cache, seqs, w.qi, w.q, out, sel, ws) == msa.MSA_OK
    _flags_clear(ws)
    out.zero_()
    q_host = w.q.cpu().pin_memory()
    qi_host = w.qi.cpu()                                  # pageable
    assert _decode(lib, w, cache, seqs, w.qi, q_host, out, sel, ws) == msa.MSA_ERR_INVALID_ARG
    assert _decode(lib, w, cache, seqs, qi_host, w.q, out, sel, ws) == msa.MSA_ERR_INVALID_ARG
    k_host = w.k_data.cpu().pin_memory()
    assert _decode(lib, w, _cache_struct(w, k_data=k_host), seqs, w.qi, w.q, out, sel, ws) == \
        msa.MSA_ERR_INVALID_ARG
    lens_host = w.seq_lens.cpu().pin_memory()
    assert _decode(lib, w, cache, _seqs_struct(w, lens_host), w.qi, w.q, out, sel, ws) == \
        msa.MSA_ERR_INVALID_ARG
    ws_host = ws.cpu().pin_memory()
    assert _decode(lib, w, cache, seqs, w.qi, w.q, out, sel, ws_host) == msa.MSA_ERR_WORKSPACE
    # nothing ran: the output is untouched and no device error was recorded
    _flags_clear(ws)
    assert int(out.view(torch.int16).abs().sum()) == 0


def test_stage_calls_reject_host_buffers(lib, wl):
    w = wl
    out, sel, ws = _buffers(w)
    cache, seqs = _cache_struct(w), _seqs_struct(w)
    bs = torch.empty(w.batch, w.q_tokens, 4, w.max_pages, device="cuda")
    qi_host = w.qi.cpu().pin_memory()
    r = lib.msa_indexer_score(ctypes.byref(cache), ctypes.byref(seqs), _vp(qi_host), w.s_qi, None,
                              _vp(bs), _vp(ws), ws.numel(), None)
    assert r == msa.MSA_ERR_INVALID_ARG
    bs_host = bs.cpu().pin_memory()
    r = lib.msa_indexer_score(ctypes.byref(cache), ctypes.byref(seqs), _vp(w.qi), w.s_qi, None,
                              _vp(bs_host), _vp(ws), ws.numel(), None)
    assert r == msa.MSA_ERR_INVALID_ARG
    sel_host = sel.cpu().pin_memory()
    r = lib.msa_sparse_attn_decode(ctypes.byref(cache), ctypes.byref(seqs), _vp(w.q), w.s_q,
                                   _vp(sel_host), w.softmax_scale, _vp(out), _vp(ws), ws.numel(), None)
    assert r == msa.MSA_ERR_INVALID_ARG
    r = lib.msa_block_maxpool_topk(_vp(bs), 0, ctypes.byref(seqs), _vp(sel_host), _vp(ws), ws.numel(), None)
    assert r == msa.MSA_ERR_INVALID_ARG
    _flags_clear(ws)


def test_kv_insert_rejects_host_buffers(lib, wl):
    w = wl
    _, _, ws = _buffers(w)
    cache, seqs = _cache_struct(w), _seqs_struct(w)
    g = torch.Generator(device="cuda").manual_seed(5)
    k_new = torch.randn(w.batch, w.q_tokens, 4, 128, generator=g, device="cuda").to(torch.bfloat16)
    v_new = torch.randn(w.batch, w.q_tokens, 4, 128, generator=g, device="cuda").to(torch.bfloat16)
    i_new = torch.randn(w.batch, w.q_tokens, 128, generator=g, device="cuda").to(torch.bfloat16)
    k_host = k_new.cpu().pin_memory()
    before = w.k_data.clone()
    r = lib.msa_kv_insert(ctypes.byref(cache), ctypes.byref(seqs), _vp(k_host), _vp(v_new), _vp(i_new),
                          _vp(ws), ws.numel(), None)
    assert r == msa.MSA_ERR_INVALID_ARG
    v_host_cache = w.v_data.cpu().pin_memory()
    r = lib.msa_kv_insert(ctypes.byref(_cache_struct(w, v_data=v_host_cache)), ctypes.byref(seqs),
                          _vp(k_new), _vp(v_new), _vp(i_new), _vp(ws), ws.numel(), None)
    assert r == msa.MSA_ERR_INVALID_ARG
    _flags_clear(ws)
    assert torch.equal(before, w.k_data)


def test_pools_shorter_than_the_page_count(lib, wl):
    """A cache descriptor that claims far more pages than its pools hold: the
    last byte of each claimed pool lies beyond device memory.  (Every page
    id in the page table is a real page, so the call would read only real
    pages even if the check let it through.)"""
    w = wl
    out, sel, ws = _buffers(w)
    cache = _cache_struct(w)
    cache.num_pages = 1 << 20          # 8 GiB of index-key codes and 32 GiB of K codes claimed
    assert w.idx_data.numel() < cache.num_pages * 128 * 64
    assert int(w.page_table.max()) < w.k_data.shape[0]
    assert _decode(lib, w, cache, _seqs_struct(w), w.qi, w.q, out, sel, ws) == msa.MSA_ERR_INVALID_ARG
    _flags_clear(ws)


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs two visible GPUs")
def test_two_devices_in_one_process(lib):
    """The per-device launch set-up (shared-memory limit, grid size): the
    same decode on device 0 and then device 1 from one process gives the
    same bits."""
    res = []
    for d in (0, 1):
        with torch.cuda.device(d):
            w = synth.make_workload("two_dev", 2, [5000, 2100], 8, paged=True, seed=62,
                                    device="cuda:%d" % d)
            cache, seqs = msa.cache_of(w), msa.seqs_of(w)
            ws = msa.alloc_workspace(seqs, device="cuda:%d" % d)
            out = torch.empty(w.batch, w.q_tokens, 64, 128, dtype=torch.bfloat16, device="cuda:%d" % d)
            sel = torch.empty(w.batch, w.q_tokens, 4, 16, dtype=torch.int32, device="cuda:%d" % d)
            msa.msa_decode(cache, seqs, w.qi, w.s_qi, w.q, w.s_q, w.softmax_scale, out, sel, ws)
            torch.cuda.synchronize(d)
            assert msa.msa_get_last_error(ws)[0] == msa.MSA_OK
            res.append((out.cpu(), sel.cpu()))
    assert torch.equal(res[0][1], res[1][1])
    assert torch.equal(res[0][0].view(torch.int16), res[1][0].view(torch.int16))


def test_launch_limits_follow_the_largest_call(lib):
    """The indexer's shared memory grows with the batch; a small call after a
    large one must not lower the kernel's limit below what the next large
    call needs."""
    big = synth.make_workload("lim_big", 6, [3000, 900, 5000, 2100, 300, 4000], 2, paged=True,
                              seed=63, device="cuda")
    small = synth.make_workload("lim_small", 1, [1000], 2, paged=True, seed=64, device="cuda")
    for w in (big, small, big, small, big):
        cache, seqs = msa.cache_of(w), msa.seqs_of(w)
        ws = msa.alloc_workspace(seqs)
        bs = torch.empty(w.batch, w.q_tokens, 4, w.max_pages, device="cuda")
        msa.msa_indexer_score(cache, seqs, w.qi, w.s_qi, None, bs, ws)
        torch.cuda.synchronize()
        assert msa.msa_get_last_error(ws)[0] == msa.MSA_OK
