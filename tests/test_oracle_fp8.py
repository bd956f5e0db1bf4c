"""Pins of the oracle's fp8 (e4m3) reading: every one of the 256 codes against
torch's float8_e4m3fn conversion, and hand values from the format's definition
(sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals at 2^-9 steps,
448 the largest value, S.1111.111 NaN)."""
import math

import numpy as np
import torch

import oracle


def test_all_codes_match_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).float().numpy()
    got = oracle.to_f32(codes.view(torch.float8_e4m3fn)).ravel()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_hand_values():
    def val(code):
        return float(oracle.to_f32(np.array([code], np.uint8))[0])
    assert val(0x38) == 1.0                      # e = 7, m = 0
    assert val(0x3c) == 1.5                      # m = 4: 1 + 4/8
    assert val(0xb8) == -1.0
    assert val(0x7e) == 448.0                    # e = 15, m = 6: 2^8 * 1.75
    assert val(0x01) == 2.0 ** -9                # smallest subnormal
    assert val(0x07) == 7 * 2.0 ** -9            # largest subnormal
    assert val(0x08) == 2.0 ** -6                # smallest normal
    assert val(0x80) == 0.0 and math.copysign(1.0, val(0x80)) == -1.0
    assert math.isnan(val(0x7f)) and math.isnan(val(0xff))
