"""Pins of the oracle's FP8 E4M3 decoder (CPU).

The decoder is written from the format definition (sign, 4-bit exponent with
bias 7, 3-bit mantissa, subnormals, S.1111.111 = NaN, no infinity); it is
checked against hand-worked codes and against torch's float8_e4m3fn, a
library implementation of the same format, on all 256 codes.
"""
import math

import torch


def test_e4m3_hand_values(orc):
    codes = torch.tensor([0x00, 0x80, 0x38, 0xB8, 0x7E, 0xFE, 0x01, 0x07, 0x08, 0x3C, 0x40, 0x46],
                         dtype=torch.uint8)
    want = [0.0, -0.0, 1.0, -1.0, 448.0, -448.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.5, 2.0, 3.5]
    got = orc.e4m3_decode(codes).tolist()
    for g, w in zip(got, want):
        assert g == w and math.copysign(1.0, g) == math.copysign(1.0, w)
    assert all(math.isnan(x) for x in orc.e4m3_decode(torch.tensor([0x7F, 0xFF], dtype=torch.uint8)).tolist())


def test_e4m3_all_codes_match_library(orc):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ours = orc.e4m3_decode(codes)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float64)
    nan = torch.isnan(lib)
    assert torch.equal(torch.isnan(ours), nan)
    assert torch.equal(ours[~nan], lib[~nan])


def test_e4m3_scale_is_exact(orc):
    codes = torch.arange(0, 126, dtype=torch.int32).to(torch.uint8)
    s = 0.0123456789
    s32 = float(torch.tensor(s, dtype=torch.float32))
    got = orc.e4m3_decode(codes, s32)
    assert torch.equal(got, orc.e4m3_decode(codes) * s32)
    assert torch.equal(got / s32, orc.e4m3_decode(codes))
