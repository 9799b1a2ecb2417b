"""Pins for the oracle's number formats (CPU only).

* hand-worked NVFP4 element decodes (golden/nvfp4_e4m3_hand_cases.txt);
* the E2M1 table of OCP MX v1.0 (golden/e2m1_values.txt);
* all 256 E4M3 bytes against torch's float8_e4m3fn decode (library);
* all 256 scales x 16 codes against torch's float8 cast of the exact product
  (library round-to-nearest-even, clamped first because torch's cast does not
  saturate);
* a whole packed row: nibble order (element 2i low nibble of byte i) and the
  scale assignment (scale s covers elements 16s..16s+15).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests import torch_ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _hand_cases():
    out = []
    for line in open(os.path.join(GOLDEN, "nvfp4_e4m3_hand_cases.txt")):
        body = line.split("#")[0].strip()
        if body:
            c, s, e = (int(x, 0) for x in body.split())
            out.append((c, s, e, line.split("#", 1)[1].strip() if "#" in line else ""))
    return out


@pytest.mark.parametrize("code,scale,expected,why", _hand_cases())
def test_hand_worked_nvfp4(code, scale, expected, why):
    prod = oracle.e2m1(code) * oracle.e4m3(scale)
    got = oracle.e4m3_round(prod)
    assert got == expected, why
    v = oracle.nvfp4_elem(code, scale)
    assert v == oracle.e4m3(expected) or (v == 0 and oracle.e4m3(expected) == 0)


def test_e2m1_table():
    t = torch_ref.e2m1_table()
    for c in range(16):
        got = oracle.e2m1(c)
        assert got == t[c].item()
        assert math.copysign(1.0, got) == math.copysign(1.0, t[c].item())


def test_e4m3_decode_all_bytes_vs_torch():
    ref = torch_ref.e4m3_to_f64(torch.arange(256, dtype=torch.int32).to(torch.uint8))
    for b in range(256):
        got = oracle.e4m3(b)
        r = ref[b].item()
        if math.isnan(r):
            assert math.isnan(got), hex(b)
        else:
            assert got == r, hex(b)
    # structural facts of the format
    assert oracle.e4m3(0x7E) == 448.0 and oracle.e4m3(0x01) == 2.0 ** -9
    assert oracle.e4m3(0x08) == 2.0 ** -6 and math.isnan(oracle.e4m3(0x7F))


def test_e4m3_round_exhaustive_products_vs_torch():
    """Every (scale byte, code) pair: the oracle's re-rounding equals torch's
    float8 cast of the exactly representable product (after clamping to the
    E4M3 range, i.e. saturation)."""
    t = torch_ref.e2m1_table()
    scales = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    sv = torch_ref.e4m3_to_f64(scales)
    for s in range(256):
        if math.isnan(sv[s].item()):
            continue
        prods = t * sv[s]
        ref = torch_ref.round_e4m3_sat(prods)
        for c in range(16):
            got = oracle.nvfp4_elem(c, s)
            assert got == ref[c].item(), (hex(s), c, prods[c].item(), got, ref[c].item())


def test_e4m3_round_grid_fixed_points_and_midpoints():
    """Every finite E4M3 value rounds to itself; every midpoint between two
    neighbours rounds to the neighbour with the even mantissa; beyond 448
    saturates."""
    vals = sorted({oracle.e4m3(b) for b in range(0x00, 0x7F)})  # non-negative finite
    for v in vals:
        assert oracle.e4m3(oracle.e4m3_round(v)) == v
        assert oracle.e4m3(oracle.e4m3_round(-v)) == -v
    for a, b in zip(vals[:-1], vals[1:]):
        mid = (a + b) / 2
        r = oracle.e4m3_round(mid)
        assert oracle.e4m3(r) in (a, b)
        assert (r & 1) == 0, (a, b, hex(r))
    for x in (448.0, 449.0, 464.0, 500.0, 1e9, float("inf")):
        assert oracle.e4m3_round(x) == 0x7E
        assert oracle.e4m3_round(-x) == 0xFE


def test_packed_row_nibble_order_and_scales():
    rng = np.random.default_rng(7)
    data = rng.integers(0, 256, 64, dtype=np.uint8)
    scale = rng.integers(0x30, 0x50, 8, dtype=np.uint8)
    got = oracle.decode_nvfp4_row(data, scale)
    ref = torch_ref.decode_nvfp4(torch.from_numpy(data), torch.from_numpy(scale)).numpy()
    assert np.array_equal(got, ref)
    # element 2i is the low nibble, 2i+1 the high nibble; scale byte d//16
    for d in (0, 1, 2, 15, 16, 17, 63, 64, 126, 127):
        code = (data[d // 2] >> 4) if d % 2 else (data[d // 2] & 15)
        assert got[d] == oracle.nvfp4_elem(int(code), int(scale[d // 16]))
