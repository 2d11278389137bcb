"""The 8-bit inputs: OCP FP8 E4M3 (torch.float8_e4m3fn) as the GPU reads it.

The forward on 8-bit inputs is compared with the fp64 oracle fed the decoded
inputs, so the decoding itself is pinned here to the format's definition:
sign bit, 4 exponent bits with bias 7, 3 mantissa bits, subnormals at
exponent field 0, and the all-ones pattern S.1111.111 as NaN (no infinities).
The rounding of the seeded draws to E4M3 is round-to-nearest-even, checked on
values halfway between neighbours.
"""
import math

import numpy as np
import torch

import attn_inputs


def e4m3_value(byte: int) -> float:
    """The value an E4M3 byte encodes, from the format's definition."""
    s = -1.0 if byte & 0x80 else 1.0
    e = (byte >> 3) & 0xF
    m = byte & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return s * m * 2.0 ** -9           # subnormal: m/8 * 2^(1-7)
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def test_every_byte_decodes_to_its_definition():
    raw = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn)
    got = raw.to(torch.float64).numpy()
    for b in range(256):
        want = e4m3_value(b)
        if math.isnan(want):
            assert math.isnan(got[b]), b
        else:
            assert got[b] == want, (b, got[b], want)
    # the landmarks: 1.0, the largest finite value 448, the smallest subnormal 2^-9
    assert e4m3_value(0x38) == 1.0 and e4m3_value(0x7E) == 448.0 and e4m3_value(0x01) == 2.0 ** -9


def test_draws_round_to_nearest_even():
    # between 1 and 2 the spacing is 1/8; a value halfway between two codes
    # goes to the one with an even mantissa
    x = torch.tensor([1.0625, 1.1875, 1.0624, 1.0626, -3.25 - 1 / 16], dtype=torch.float32)
    got = x.to(torch.float8_e4m3fn).to(torch.float64).tolist()
    assert got == [1.0, 1.25, 1.0, 1.125, -3.25]


def test_fp8_draws_are_the_rounded_fp32_draws():
    (q8,) = attn_inputs.draw(1, 64, 2, 128, "fp8", 77, 1)
    (q32,) = attn_inputs.draw_fp32(1, 64, 2, 128, 77, 1)
    assert q8.dtype == torch.float8_e4m3fn
    dec = attn_inputs.to_f64(q8)
    # every draw within half a code spacing (2^-4 relative, 2^-10 absolute below 2^-6)
    tol = np.maximum(np.abs(q32.astype(np.float64)) * 2.0 ** -4, 2.0 ** -10)
    assert np.all(np.abs(dec - q32) <= tol)
