"""Pins of the oracle's exact widening of the storage formats, against bit
patterns worked out by hand from the IEEE layouts (not from the oracle).

bf16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits; a normal value
is (-1)^s * 2^(e - 127) * (1 + f / 128), a subnormal (e = 0) is
(-1)^s * 2^-126 * f / 128.  binary16: 5 exponent bits (bias 15), 10 fraction
bits, subnormals (-1)^s * 2^-14 * f / 1024.  Every parity test widens the
CUDA path's bf16 output and the synthetic fp16 scales with these functions,
so a mistake here would otherwise show only as a GPU parity failure.
"""
import math

import numpy as np
import pytest

import oracle

BF16 = [
    (0x3F80, 1.0),                              # s 0, e 127, f 0
    (0xBF80, -1.0),
    (0xC020, -2.5),                             # s 1, e 128, f 0x20: -2 * (1 + 32/128)
    (0x4049, 3.140625),                         # e 128, f 0x49 = 73: 2 * (1 + 73/128)
    (0x3E80, 0.25),                             # e 125
    (0x0001, 2.0 ** -133),                      # smallest subnormal: 2^-126 * 1/128
    (0x807F, -(127 / 128) * 2.0 ** -126),       # largest negative subnormal
    (0x0080, 2.0 ** -126),                      # smallest normal
    (0x7F7F, (2 - 2.0 ** -7) * 2.0 ** 127),     # largest finite
    (0x0000, 0.0),
    (0x7F80, math.inf),
    (0xFF80, -math.inf),
]


@pytest.mark.parametrize("bits,value", BF16)
def test_bf16_patterns(bits, value):
    got = oracle.bf16_bits_to_f64(np.array([bits], dtype=np.uint16))
    assert got.dtype == np.float64
    assert got[0] == value


def test_bf16_negative_zero_and_nan():
    z = oracle.bf16_bits_to_f64(np.array([0x8000], dtype=np.uint16))[0]
    assert z == 0.0 and math.copysign(1.0, z) == -1.0
    assert math.isnan(oracle.bf16_bits_to_f64(np.array([0x7FC0], dtype=np.uint16))[0])


@pytest.mark.filterwarnings("ignore:invalid value encountered in cast:RuntimeWarning")
def test_bf16_every_pattern_by_the_formula():
    """All 65536 patterns against the layout formula evaluated with exact
    powers of two (NaN patterns excepted, which must come out NaN)."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    got = oracle.bf16_bits_to_f64(bits.astype(np.uint16))
    s, e, f = bits >> 15, (bits >> 7) & 0xFF, bits & 0x7F
    sign = np.where(s == 1, -1.0, 1.0)
    normal = np.ldexp(1.0 + f / 128.0, e.astype(np.int64) - 127)
    sub = np.ldexp(f / 128.0, -126)
    want = sign * np.where(e == 0, sub, normal)
    want = np.where((e == 255) & (f == 0), sign * np.inf, want)
    nan = (e == 255) & (f != 0)
    assert np.all(np.isnan(got[nan]))
    assert np.array_equal(got[~nan], want[~nan])


F16 = [(0x3C00, 1.0), (0xC100, -2.5), (0x7BFF, 65504.0), (0x0001, 2.0 ** -24), (0x0400, 2.0 ** -14),
       (0x3555, 1365 / 4096)]  # e 13, f 0x155 = 341: 2^-2 * (1 + 341/1024)


@pytest.mark.parametrize("bits,value", F16)
def test_f16_patterns(bits, value):
    got = oracle.f16_to_f64(np.array([bits], dtype=np.uint16).view(np.float16))
    assert got.dtype == np.float64 and got[0] == value
