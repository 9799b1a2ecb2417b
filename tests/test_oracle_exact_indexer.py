"""Pins of the oracle's exact index-key mode (NVFP4 keys scored at
e2m1(code) * e4m3(scale) * s_idx, without the E4M3 re-rounding: the FP16
scoring of [post, "NVIDIA Rubin optimized MSA"]).

Independent of the oracle's own arithmetic:
  * hand-worked products where the re-rounding changes the value (the same
    (code, scale) pairs as the re-rounding pins, now expected unrounded);
  * a basis-vector probe that reads every key element back through the score,
    against the OCP E2M1 grid and torch's float8 decode of the scale byte;
  * with power-of-two scale bytes every product already lies on the E4M3
    grid, so the exact mode must equal the re-rounded mode there;
  * everywhere, exact and re-rounded scores differ by at most the E4M3
    half-step of each key element (2^-4 relative) times |q|.
"""
import numpy as np
import pytest
import torch

import oracle

E2M1_GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]     # OCP MX v1.0 magnitudes


def e2m1_ref(code: int) -> float:
    v = E2M1_GRID[code & 7]
    return -v if code & 8 else v


def e4m3_ref(byte: int) -> float:
    return float(torch.tensor([byte], dtype=torch.uint8).view(torch.float8_e4m3fn).double())


def one_page_cache(codes, scales, exact, seq_len=128):
    """One sequence on one page: codes [128][128] nibble values, scales [128][8]."""
    codes = np.asarray(codes, np.uint8)
    data = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8).reshape(1, 128, 64)
    z = lambda *s: np.zeros(s, np.uint8)
    return oracle.Cache(idx_data=np.ascontiguousarray(data),
                        idx_scale=np.ascontiguousarray(np.asarray(scales, np.uint8).reshape(1, 128, 8)),
                        k_data=z(1, 4, 128, 64), k_scale=z(1, 4, 128, 8), v_data=z(1, 4, 128, 64),
                        v_scale=z(1, 4, 128, 8), s_idx=1.0, s_k=1.0, s_v=1.0, page_table=None,
                        max_pages=1, seq_lens=np.array([seq_len], np.int32), q_tokens=1,
                        idx_exact=exact)


def basis_queries(dims):
    """qi [1][1][4][128]: E4M3 1.0 (0x38) at dims[g] for group g, 0 elsewhere."""
    qi = np.zeros((1, 1, 4, 128), np.uint8)
    for g, d in enumerate(dims):
        qi[0, 0, g, d] = 0x38
    return qi


# (code, scale byte, exact product, E4M3 re-rounded product)
HAND = [(0x3, 0x39, 1.6875, 1.75), (0x3, 0x3B, 2.0625, 2.0), (0x3, 0x3D, 2.4375, 2.5),
        (0x5, 0x3F, 5.625, 5.5), (0x7, 0x38, 6.0, 6.0), (0xB, 0x39, -1.6875, -1.75)]


@pytest.mark.parametrize("code,sb,exact,rerounded", HAND)
def test_hand_worked_products(code, sb, exact, rerounded):
    codes = np.zeros((128, 128), np.uint8)
    scales = np.full((128, 8), 0x38, np.uint8)
    codes[0, 0] = code
    scales[0, 0] = sb
    qi = basis_queries([0, 0, 0, 0])
    for mode, want in ((True, exact), (False, rerounded)):
        c = one_page_cache(codes, scales, mode, seq_len=1)
        ts, bs = oracle.indexer(c, qi, 1.0, [(0, 0)])
        assert ts[0, 0, 0] == want and bs[0, 0, 0] == want, (mode, ts[0, 0, 0], want)


def test_basis_probe_reads_every_element():
    rng = np.random.default_rng(41)
    codes = rng.integers(0, 16, size=(128, 128))
    scales = rng.integers(0, 0x7F, size=(128, 8))          # every finite non-negative byte range
    scales[rng.random((128, 8)) < 0.2] |= 0x80              # and some negative scales
    scales[scales == 0xFF] = 0xFE
    c = one_page_cache(codes, scales, True)
    s_qi = 0.75
    for dims in ([0, 1, 16, 127], [15, 31, 64, 100], [2, 47, 80, 113]):
        ts, _ = oracle.indexer(c, basis_queries(dims), s_qi, [(0, 0)])
        for g, d in enumerate(dims):
            want = [s_qi * e2m1_ref(int(codes[j, d])) * e4m3_ref(int(scales[j, d // 16]))
                    for j in range(128)]
            np.testing.assert_array_equal(ts[0, g, :128], np.array(want))


def test_power_of_two_scales_match_rerounded_mode():
    rng = np.random.default_rng(43)
    codes = rng.integers(0, 16, size=(128, 128))
    scales = rng.choice([0x28, 0x30, 0x38, 0x40, 0x48, 0xB8], size=(128, 8))   # +-2^k
    qi = rng.integers(0, 0x7F, size=(1, 1, 4, 128)).astype(np.uint8)
    qi[rng.random(qi.shape) < 0.5] |= 0x80
    qi[qi == 0xFF] = 0xFE
    ex = oracle.indexer(one_page_cache(codes, scales, True), qi, 1.0, [(0, 0)])
    rr = oracle.indexer(one_page_cache(codes, scales, False), qi, 1.0, [(0, 0)])
    np.testing.assert_array_equal(ex[0][:, :, :128], rr[0][:, :, :128])
    np.testing.assert_array_equal(ex[1], rr[1])


def test_exact_and_rerounded_differ_within_half_step():
    rng = np.random.default_rng(47)
    codes = rng.integers(0, 16, size=(128, 128))
    scales = rng.integers(0x20, 0x60, size=(128, 8))
    qi = rng.integers(0, 0x7F, size=(1, 1, 4, 128)).astype(np.uint8)
    qv = np.array([[e4m3_ref(int(b)) for b in row] for row in qi[0, 0]])
    kabs = np.array([[abs(e2m1_ref(int(codes[j, d])) * e4m3_ref(int(scales[j, d // 16])))
                      for d in range(128)] for j in range(128)])
    ex, _ = oracle.indexer(one_page_cache(codes, scales, True), qi, 1.0, [(0, 0)])
    rr, _ = oracle.indexer(one_page_cache(codes, scales, False), qi, 1.0, [(0, 0)])
    bound = (np.abs(qv) @ kabs.T) * 2.0 ** -4                # [4][128]
    diff = np.abs(ex[0, :, :128] - rr[0, :, :128])
    assert np.all(diff <= bound * (1 + 1e-12))
    assert diff.max() > 0                                    # the modes really differ
