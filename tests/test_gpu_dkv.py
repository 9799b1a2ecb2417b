"""GPU parity of the decode-once attention: when every (sequence, group)
selects each of its blocks several times over (T x 16 >= 4 x max_pages, as in
prefill), the step decodes every visible block's K and V to E4M3 once into
the workspace and the attention loads those rows instead of decoding per
(token, group) ([post, "AMD GPU support", "NVFP4 MSA kernel"]: dequantise a
page once for the requests that read it; [post, "NVIDIA Blackwell optimized
MSA kernels"]: the E4M3 re-rounding of the NVFP4 cache feeds FP8 MMA).

Checked against the float64 oracle over the GPU's own selection, and bit for
bit against the same step run without the decode-once rows (the 16 MiB
fixed scratch of msa_decode_static, which cannot hold them: the attention
then decodes per item) -- the same E4M3 operands and the same MMAs."""
import ctypes
import zlib

import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_decode_b200 as msa
from block_sparse_attention_decode_b200 import build as msa_build
from block_sparse_attention_decode_b200 import synth
from tests import parity

pytestmark = pytest.mark.gpu

# (name, lengths, query tokens): small contexts with many query tokens each,
# so that T x 16 >= 4 x max_pages; the decode-once rows (B x max_pages x
# 128 KB) exceed the 16 MiB fixed scratch while the rest of the step fits it
CASES = [
    ("t64_two", [5000, 9000], 64),
    ("t128_ragged", [2100, 16000, 700], 128),
]


@pytest.fixture(scope="module")
def lib():
    msa_build.build()
    return msa.load()


def _workload(name, lens, T):
    return synth.make_workload(name, len(lens), lens, T, paged=True,
                               seed=zlib.crc32(name.encode()) % 10000, device="cuda")


def _static(lib, cache, seqs, w, out, sel):
    return lib.msa_decode_static(ctypes.byref(cache.c), ctypes.byref(seqs.c),
                                 ctypes.c_void_p(w.qi.data_ptr()), w.s_qi,
                                 ctypes.c_void_p(w.q.data_ptr()), w.s_q, w.softmax_scale,
                                 ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(sel.data_ptr()),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("name,lens,T", CASES, ids=[c[0] for c in CASES])
def test_decode_once_matches_oracle_and_per_item_decode(lib, name, lens, T):
    w = _workload(name, lens, T)
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    dkv = w.batch * w.max_pages * 4 * 2 * 128 * 128
    assert T * 16 >= 4 * w.max_pages
    assert msa.msa_workspace_size(seqs) >= dkv
    assert msa.msa_workspace_size(seqs) > msa.STATIC_WORKSPACE_BYTES       # static runs without it
    ws = msa.alloc_workspace(seqs)
    out = torch.full((w.batch, T, 64, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    sel = torch.full((w.batch, T, 4, 16), -7, dtype=torch.int32, device="cuda")
    msa.msa_decode(cache, seqs, w.qi, w.s_qi, w.q, w.s_q, w.softmax_scale, out, sel, ws)
    torch.cuda.synchronize()
    assert msa.msa_get_last_error(ws)[0] == msa.MSA_OK

    # the same step without the decode-once rows: identical selection and output
    out_s = torch.full_like(out, float("nan"))
    sel_s = torch.full_like(sel, -7)
    assert _static(lib, cache, seqs, w, out_s, sel_s) == msa.MSA_OK
    torch.cuda.synchronize()
    assert torch.equal(sel, sel_s)
    assert torch.equal(out.view(torch.int16), out_s.view(torch.int16))

    # against the oracle, over the GPU's selection
    c, _ = parity.host_cache(w)
    rows = oracle.all_rows(c)
    _, q = parity.host_queries(w, list(range(w.batch)))
    gsel = sel.cpu().numpy().reshape(len(rows), 4, 16)
    ref = oracle.attention(c, q, w.s_q, w.softmax_scale, rows, gsel)
    parity.check_output(out.reshape(len(rows), 64, 128), ref, name)


def test_decode_once_stage_entry_point(lib):
    """msa_sparse_attn_decode alone (selection given) takes the same path."""
    w = _workload("stage_t64", [3000, 4500], 64)
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    c, _ = parity.host_cache(w)
    rows = oracle.all_rows(c)
    qi, q = parity.host_queries(w, list(range(w.batch)))
    _, rbs = oracle.indexer(c, qi, w.s_qi, rows, token_scores=False)
    rsel = oracle.select(c, rows, rbs)
    sel = torch.from_numpy(np.ascontiguousarray(rsel.reshape(w.batch, 64, 4, 16)).astype(np.int32)).cuda()
    out = torch.full((w.batch, 64, 64, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    msa.msa_sparse_attn_decode(cache, seqs, w.q, w.s_q, sel, w.softmax_scale, out, ws)
    torch.cuda.synchronize()
    assert msa.msa_get_last_error(ws)[0] == msa.MSA_OK
    ref = oracle.attention(c, q, w.s_q, w.softmax_scale, rows, rsel)
    parity.check_output(out.reshape(len(rows), 64, 128), ref, "stage entry point")
