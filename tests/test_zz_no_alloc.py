"""msa_decode_static: the decode step for callers that cannot allocate device
memory where they call it (code running under another framework's caching
allocator, plugin/custom-op execution paths that forbid allocations, hot
serving loops).  Its scratch is a fixed array inside the library, so it takes
no workspace argument.

Checked through the C ABI against msa_decode with a caller workspace, with
the tolerances the other parity tests use, on two calls in a row (the shared
array keeps the previous call's contents).  This file is collected last so a
run that stops at the first failure has run every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_decode_b200 as msa
from block_sparse_attention_decode_b200 import build as msa_build
from block_sparse_attention_decode_b200 import synth
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    msa_build.build()
    return msa.load()


def _call_static(lib, cache, seqs, w, out, sel):
    return lib.msa_decode_static(ctypes.byref(cache.c), ctypes.byref(seqs.c),
                                 ctypes.c_void_p(w.qi.data_ptr()), w.s_qi,
                                 ctypes.c_void_p(w.q.data_ptr()), w.s_q, w.softmax_scale,
                                 ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(sel.data_ptr()),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_scratch_matches_caller_workspace_twice(lib):
    # a mix of sparse (> 16 blocks) and dense rows, paged, 2 query tokens;
    # small enough for the 16 MiB scratch, large enough for split-K attention
    w = synth.make_workload("static", 4, [40000, 2300, 1000, 70001], 2, paged=True, seed=71,
                            device="cuda")
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    assert msa.msa_workspace_size(seqs) <= msa.STATIC_WORKSPACE_BYTES
    ws = msa.alloc_workspace(seqs)
    out_ref = torch.empty(w.batch, w.q_tokens, 64, 128, dtype=torch.bfloat16, device="cuda")
    sel_ref = torch.empty(w.batch, w.q_tokens, 4, 16, dtype=torch.int32, device="cuda")
    msa.msa_decode(cache, seqs, w.qi, w.s_qi, w.q, w.s_q, w.softmax_scale, out_ref, sel_ref, ws)
    torch.cuda.synchronize()
    assert msa.msa_get_last_error(ws)[0] == msa.MSA_OK
    ref = out_ref.float().cpu().numpy().astype(np.float64)
    for call in range(2):
        out = torch.full_like(out_ref, float("nan"))
        sel = torch.full_like(sel_ref, -7)
        assert _call_static(lib, cache, seqs, w, out, sel) == msa.MSA_OK, call
        torch.cuda.synchronize()
        assert torch.equal(sel, sel_ref), call
        parity.check_output(out, ref, "static scratch, call %d" % call)


def test_static_scratch_rejects_batches_beyond_its_size(lib):
    # 8 sequences x 256 query tokens x 1,024 blocks need 32 MiB of block
    # scores alone: more than the fixed scratch holds.  The size check comes
    # first, so the call returns before touching any tensor.
    lens = torch.full((8,), 131072, dtype=torch.int32, device="cuda")
    seqs = msa.Seqs(lens, 256, 1024)
    assert msa.msa_workspace_size(seqs) > msa.STATIC_WORKSPACE_BYTES
    w = synth.make_workload("static_small", 1, [300], 1, paged=False, seed=72, device="cuda")
    cache = msa.cache_of(w)
    dummy = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    st = lib.msa_decode_static(ctypes.byref(cache.c), ctypes.byref(seqs.c), p, 1.0, p, 1.0, 0.1,
                               p, None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == msa.MSA_ERR_WORKSPACE
