"""Pins of the oracle's cache-insert encoder (NVFP4 / FP8), independent of its
own arithmetic: grid values must come back exactly, every code must be a
nearest representable value (brute force over all codes), the scale byte
and the FP8 keys must equal torch's float8 cast of the same fp32 quotient,
midpoint ties go to the even code, and inserted rows land in the page and
slot of their position and nowhere else.
"""
import numpy as np
import pytest
import torch

import oracle

S_TS = [6.0 / 448.0, 1.0 / 3.0, 0.0625]


def e2m1_values():
    return np.array([oracle.e2m1(c) for c in range(16)])


def test_e2m1_round_hand_cases():
    # grid points map to their own code; midpoints to the code with an even
    # mantissa bit (OCP E2M1 grid 0, 0.5, 1, 1.5, 2, 3, 4, 6)
    grid = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}
    for y, c in grid.items():
        assert oracle.e2m1_round(y) == c, y
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for y, c in ties.items():
        assert oracle.e2m1_round(y) == c, y
    assert oracle.e2m1_round(6.5) == 7 and oracle.e2m1_round(1e9) == 7     # saturates
    assert oracle.e2m1_round(1e30) == 7      # beyond where y - 4 and y - 6 are equal in f64
    assert oracle.e2m1_round(0.2499) == 0 and oracle.e2m1_round(0.2501) == 1


@pytest.mark.parametrize("s_t", S_TS)
def test_grid_values_round_trip(s_t):
    """x = e2m1(c) * e4m3(sb) * s_t with a magnitude-6 element in every block
    encodes back to exactly (c, sb) -- zero keeps code 0."""
    rng = np.random.default_rng(7)
    vals = e2m1_values()
    for trial in range(200):
        codes = rng.integers(0, 16, size=128)
        codes[::16] = rng.choice([7, 15], size=8)          # amax = 6 * scale in each block
        sb = rng.integers(1, 0x60, size=8)                 # scale bytes (subnormal ones too)
        sd = np.array([oracle.e4m3(int(b)) for b in sb])
        x = np.array([np.float32(vals[c]) * np.float32(sd[d // 16]) * np.float32(s_t)
                      for d, c in enumerate(codes)], np.float32)
        data, sc = oracle.nvfp4_encode_row(x, s_t)
        assert list(sc) == list(sb), trial
        got = np.empty(128, np.int64)
        got[0::2] = data & 15
        got[1::2] = data >> 4
        want = np.where((codes & 7) == 0, 0, codes)
        np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("s_t", S_TS)
def test_codes_are_nearest_values_and_scale_is_torch_cast(s_t):
    rng = np.random.default_rng(11)
    vals = e2m1_values()
    for trial in range(100):
        x = (rng.standard_normal(128) * rng.uniform(0.01, 50)).astype(np.float32)
        data, sc = oracle.nvfp4_encode_row(x, s_t)
        for j in range(8):
            blk = x[16 * j:16 * j + 16]
            amax = np.float32(np.abs(blk).max())
            six_st = torch.tensor([s_t], dtype=torch.float32) * 6.0          # fp32 product
            r = torch.tensor([amax], dtype=torch.float32) / six_st
            if float(r) <= 448.0:     # torch's cast does not saturate: compare in range
                assert int(r.to(torch.float8_e4m3fn).view(torch.uint8)) == int(sc[j])
            else:
                assert int(sc[j]) == 0x7E
            u = oracle.e4m3(int(sc[j])) * float(np.float32(s_t))
            for i in range(16):
                d = 16 * j + i
                c = int(data[d >> 1] >> 4) if d & 1 else int(data[d >> 1] & 15)
                dist = np.abs(blk[i] - vals * u)
                assert dist[c] <= dist.min() * (1 + 1e-6) + 1e-30, (trial, d, c)


def test_fp8_rows_equal_torch_cast():
    rng = np.random.default_rng(13)
    for s_t in (1.0 / 64.0, 0.3):
        x = (rng.standard_normal(128) * 3).astype(np.float32)
        got = oracle.fp8_encode_row(x, s_t)
        q = torch.from_numpy(x) / torch.tensor(s_t, dtype=torch.float32)
        inr = (q.abs() <= 448.0).numpy()             # torch's cast does not saturate
        want = q.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        np.testing.assert_array_equal(got[inr], want[inr])
        np.testing.assert_array_equal(got[~inr], np.where(x[~inr] < 0, 0xFE, 0x7E))


def test_saturation_and_zero_blocks():
    x = np.zeros(128, np.float32)
    x[16:32] = 1e6                                    # far above 448 * 6 * s_t
    x[32:48] = 1e30                                   # quotients far beyond f64 resolution of 6
    data, sc = oracle.nvfp4_encode_row(x, 6.0 / 448.0)
    assert sc[0] == 0 and np.all(data[:8] == 0)          # all-zero block
    assert sc[1] == 0x7E                               # scale saturates at 448
    assert np.all(data[8:24] == 0x77)                  # codes saturate at 6
    assert sc[2] == 0x7E
    # a small negative value that rounds to magnitude 0 gets code 0, not -0
    x = np.zeros(128, np.float32)
    x[0], x[1] = 6.0, -0.1                            # scale 1, y(-0.1) -> 0
    data, sc = oracle.nvfp4_encode_row(x, 1.0)
    assert data[0] == 0x07
    x = np.full(128, -2.0, np.float32)
    data, sc = oracle.nvfp4_encode_row(x, 1.0)
    # amax 2 -> scale E4M3(1/3) = 0.34375, y = -5.8 -> code 7 with the sign
    assert sc[0] == oracle.e4m3_round(np.float32(2.0) / np.float32(6.0)) and data[0] == 0xFF


def test_insert_places_rows_by_page_table():
    rng = np.random.default_rng(17)
    B, T, mp = 2, 3, 5
    lens = np.array([300, 129], np.int32)              # positions 297..299 and 126..128
    P = B * mp
    pt = rng.permutation(P).astype(np.int32).reshape(B, mp)
    z = lambda *s: np.zeros(s, np.uint8)
    c = oracle.Cache(idx_data=z(P, 128, 64), idx_scale=z(P, 128, 8), k_data=z(P, 4, 128, 64),
                     k_scale=z(P, 4, 128, 8), v_data=z(P, 4, 128, 64), v_scale=z(P, 4, 128, 8),
                     s_idx=0.02, s_k=6 / 448, s_v=0.05, page_table=pt, max_pages=mp,
                     seq_lens=lens, q_tokens=T)
    k = rng.standard_normal((B, T, 4, 128)).astype(np.float32)
    v = rng.standard_normal((B, T, 4, 128)).astype(np.float32)
    ix = rng.standard_normal((B, T, 128)).astype(np.float32)
    assert oracle.kv_insert(c, k, v, ix) == 0
    touched = np.zeros((P, 128), bool)
    for b in range(B):
        for t in range(T):
            pos = lens[b] - T + t
            p, slot = pt[b, pos // 128], pos % 128
            touched[p, slot] = True
            for g in range(4):
                d, s = oracle.nvfp4_encode_row(k[b, t, g], 6 / 448)
                assert np.array_equal(c.k_data[p, g, slot], d) and np.array_equal(c.k_scale[p, g, slot], s)
                d, s = oracle.nvfp4_encode_row(v[b, t, g], 0.05)
                assert np.array_equal(c.v_data[p, g, slot], d) and np.array_equal(c.v_scale[p, g, slot], s)
                # the decoded row is within the NVFP4 step of the input
                dec = oracle.decode_nvfp4_row(d, s) * 0.05
                assert np.abs(dec - v[b, t, g]).max() < 0.5 * np.abs(v[b, t, g]).max()
            d, s = oracle.nvfp4_encode_row(ix[b, t], 0.02)
            assert np.array_equal(c.idx_data[p, slot], d) and np.array_equal(c.idx_scale[p, slot], s)
    # nothing else was written
    for p in range(P):
        for slot in range(128):
            if not touched[p, slot]:
                assert not c.k_data[p, :, slot].any() and not c.v_scale[p, :, slot].any()
                assert not c.idx_data[p, slot].any()
