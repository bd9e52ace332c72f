"""Pins of the oracle's NVFP4 decoder and of the seeded NVFP4 input recipe (CPU).

The decoder is written from the format definitions (FP4 E2M1 elements, E4M3
block scales over 16 consecutive elements, an fp32 per-tensor scale); it is
checked against values worked by hand in tests/golden/nvfp4_hand_values.json
(every element code, the nibble order, a row with two different block
scales), so that a wrong exponent bias, a swapped nibble or a block index
taken along the wrong axis each fail a test.  The input recipe (synth.to_nvfp4)
is checked for what a quantiser must satisfy: values on the grid come back
unchanged, every element lands within half a grid step of its input, and a
second pass changes nothing.
"""
import json
import math
import os

import torch

from block_causal_linear_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "nvfp4_hand_values.json")))


def same(a, b):
    return a == b and math.copysign(1.0, a) == math.copysign(1.0, b)


def test_e2m1_every_code(orc):
    got = orc.e2m1_decode(torch.arange(16)).tolist()
    assert all(same(g, w) for g, w in zip(got, GOLD["e2m1"]))


def test_nibble_order(orc):
    got = orc.nvfp4_decode(torch.tensor([[0x2A] * 8], dtype=torch.uint8), torch.tensor([[0x38]], dtype=torch.uint8))
    assert got[0, :2].tolist() == GOLD["byte_0x2A"]


def test_row_with_two_block_scales(orc):
    codes = torch.tensor([GOLD["row_codes"]], dtype=torch.uint8)
    sf = torch.tensor([GOLD["row_block_scales"]], dtype=torch.uint8)
    got = orc.nvfp4_decode(codes, sf, GOLD["row_tensor_scale"])
    assert got[0].tolist() == GOLD["row_values"]


def test_block_scale_follows_the_last_axis(orc):
    # [2 rows][32 elements]: each row has its own two block scales
    codes = torch.full((2, 16), 0x22, dtype=torch.uint8)            # every element 1.0
    sf = torch.tensor([[0x38, 0x40], [0x30, 0x48]], dtype=torch.uint8)   # 1, 2 | 0.5, 4
    got = orc.nvfp4_decode(codes, sf)
    want = torch.tensor([[1.0] * 16 + [2.0] * 16, [0.5] * 16 + [4.0] * 16], dtype=torch.float64)
    assert torch.equal(got, want)


def test_quantiser_keeps_grid_values(orc):
    g = torch.Generator().manual_seed(3)
    codes = torch.randint(0, 256, (4, 7, 16), generator=g, dtype=torch.int32).to(torch.uint8)
    sf = torch.randint(0x20, 0x50, (4, 7, 2), generator=g, dtype=torch.int32).to(torch.uint8)
    # one block reaches 6 * 448 * 0.125: the recipe's tensor scale is then 0.125
    # again and every block scale reappears exactly
    codes[0, 0, 0], sf[0, 0, 0] = 0x77, 0x7E
    x = orc.nvfp4_decode(codes, sf, 0.125)
    c2, sf2, s2 = synth.to_nvfp4(x)
    assert s2 == 0.125
    back = orc.nvfp4_decode(c2, sf2, s2)
    # a block whose largest magnitude is 6 * scale is representable exactly
    exact = x.reshape(4, 7, 2, 16).abs().amax(-1) == orc.e4m3_decode(sf) * 0.125 * 6
    xb, bb = x.reshape(4, 7, 2, 16), back.reshape(4, 7, 2, 16)
    assert torch.equal(xb[exact], bb[exact])


def test_quantiser_error_bound_and_idempotence(orc):
    x = torch.randn(3, 50, 4, 32, generator=torch.Generator().manual_seed(11), dtype=torch.float64)
    codes, sf, s = synth.to_nvfp4(x)
    dec = orc.nvfp4_decode(codes, sf, s)
    step = orc.e4m3_decode(sf).repeat_interleave(16, -1) * s   # one unit of the E2M1 grid
    # half the widest grid step (2 units, between 4 and 6), plus the overshoot
    # of a block scale rounded down by at most 2^-4 relative (6 * 2^-4 units)
    assert bool(((dec - x).abs() <= step * (1.0 + 6.0 / 16.0)).all())
    assert torch.equal(torch.sign(dec[dec != 0]), torch.sign(x[dec != 0]))
    c2, sf2, s2 = synth.to_nvfp4(dec)
    assert torch.equal(c2, codes) and torch.equal(sf2, sf) and s2 == s


def test_quantiser_zero_and_sign_cases(orc):
    codes, sf, s = synth.to_nvfp4(torch.zeros(2, 32, dtype=torch.float64))
    assert s == 1.0 and int(codes.sum()) == 0 and int(sf.sum()) == 0
    # one block of +-10.5 = 6 * 448 * 2^-8 (the tensor scale is then exactly 2^-8): element
    # codes 0x7 and 0xF (6, -6) at the largest block scale; an all-zero block gets scale 0
    x = torch.tensor([[10.5, -10.5] * 8 + [0.0] * 16], dtype=torch.float64)
    codes, sf, s = synth.to_nvfp4(x)
    assert s == 2.0 ** -8
    assert codes[0, :8].tolist() == [0xF7] * 8 and sf[0, 0] == 0x7E and sf[0, 1] == 0x00
    assert torch.equal(orc.nvfp4_decode(codes, sf, s), x)
