"""GPU parity on the full-size workloads, in the launch configuration the
benchmark times (msa_decode over the whole batch), checked on sampled
sequences and tokens that the oracle computes one by one.

Workloads (seeded, synthetic, N(0,1) before quantisation):
  ctx4k_b1_t1          1 x 4,096 tokens, 1 query token, contiguous
  ctx32k_b32_t1        32 x 32,768, contiguous, 1 in 64 blocks planted +3 sigma
  ctx32k_b32_t1_fp8idx same with FP8 index keys
  ctx128k_b64_t8       64 x 131,072, 8 query tokens (causal), shuffled pages
  ragged_b16_t1        16 ragged lengths in [2,048, 262,144], shuffled pages
  prefill_67584_t2048  1 x (65,536 cached + 2,048 new), 2,048 query tokens
and the 128K workload once more with exactly scored index keys.
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_decode_b200 as msa
from block_sparse_attention_decode_b200 import build as msa_build
from block_sparse_attention_decode_b200 import synth
from tests import parity
from tests.test_gpu_parity import compare_decode

pytestmark = pytest.mark.gpu

SAMPLES = {
    "ctx4k_b1_t1": ([0], None),
    "ctx32k_b32_t1": ([0, 17, 31], None),
    "ctx32k_b32_t1_fp8idx": ([3, 30], None),
    "ctx128k_b64_t8": ([5, 63], None),
    "ragged_b16_t1": ([0, 1, 2, 9], None),
    "prefill_67584_t2048": ([0], [0, 1, 127, 128, 1000, 2047]),
}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    msa_build.build()
    msa.load()


@pytest.mark.parametrize("name", list(SAMPLES))
def test_full_size_sampled(name):
    torch.cuda.empty_cache()
    w = synth.workload(name, device="cuda")
    seq_ids, tokens = SAMPLES[name]
    if name == "ragged_b16_t1":
        lens = w.seq_lens.cpu().tolist()
        seq_ids = sorted(set(seq_ids + [int(np.argmax(lens))]))
    swaps, mx, mean = compare_decode(w, seq_ids, tokens, what=name)
    print("%s: near-tie swaps %d, max-abs %.3g, mean-abs %.3g" % (name, swaps, mx, mean))
    del w
    torch.cuda.empty_cache()


def test_full_size_exact_indexer_sampled():
    """The benchmark workload with the index keys scored at their exact value
    (MSA_IDX_NVFP4_EXACT), sampled like the rest."""
    torch.cuda.empty_cache()
    w = synth.workload("ctx128k_b64_t8", device="cuda")
    w = synth.Workload(**{**w.__dict__, "idx_exact": True})
    swaps, mx, mean = compare_decode(w, [11], None, what="ctx128k_b64_t8 exact")
    print("ctx128k_b64_t8 exact: near-tie swaps %d, max-abs %.3g, mean-abs %.3g" % (swaps, mx, mean))
    del w
    torch.cuda.empty_cache()
