"""Pins for the oracle's own sign packer (CPU only).

The packed layout is the library's contract (include/lb.h): word w of a row
holds columns 32w .. 32w+31, bit j set iff column 32w + j is negative, rows
padded to a multiple of 4 words with zero bits.  The expected words here are
packed by hand in tests/golden/pack_hand.txt.
"""
import numpy as np
import pytest

import oracle
from tests.conftest import load_golden


def _u_matrix(fx):
    u = np.ones((fx["u_rows"], fx["u_cols"]), dtype=np.int8)
    for row, cols in enumerate(fx["u_negative_columns"]):
        u[row, cols] = -1
    return u


def test_ld_words():
    assert [oracle.packed_ld_words(c) for c in (1, 32, 33, 128, 129, 256, 288, 4096, 28672)] == \
        [1, 1, 2, 4, 5, 8, 9, 128, 896]


def test_hand_packed_u_and_v():
    fx = load_golden("pack_hand.txt")
    u = _u_matrix(fx)
    assert np.array_equal(oracle.pack_signs(u, "U", ld_words=4), np.array(fx["u_words"], np.uint32))
    assert np.array_equal(oracle.pack_signs(u.T.copy(), "V", ld_words=4), np.array(fx["v_words"], np.uint32))
    # float sources give the same words; the smallest stride drops the zero words
    assert np.array_equal(oracle.pack_signs(u.astype(np.float32), "U", "f32"),
                          np.array(fx["u_words"], np.uint32)[:, :2])


@pytest.mark.parametrize("dtype,key", [("f32", "special_f32_bits"), ("f16", "special_f16_bits"),
                                       ("bf16", "special_bf16_bits"), ("i8", "special_i8")])
def test_special_values(dtype, key):
    fx = load_golden("pack_hand.txt")
    if dtype == "f32":
        src = np.array(fx[key], dtype=np.uint32).view(np.float32)[None, :]
    elif dtype == "f16":
        src = np.array(fx[key], dtype=np.uint16).view(np.float16)[None, :]
    elif dtype == "bf16":
        src = np.array(fx[key], dtype=np.uint16)[None, :]
    else:
        src = np.array(fx[key], dtype=np.int8)[None, :]
    words = oracle.pack_signs(src, "U", dtype, ld_words=4)
    assert words.shape == (1, 4)
    assert int(words[0, 0]) == fx["special_word0"]
    assert not words[0, 1:].any()
    assert oracle.pack_signs(src, "U", dtype).shape == (1, 1)


@pytest.mark.parametrize("rows,cols", [(3, 1), (5, 31), (4, 33), (2, 100), (7, 256)])
def test_round_trip_and_zero_padding(rows, cols):
    rng = np.random.default_rng(rows * 1000 + cols)
    s = (1 - 2 * rng.integers(0, 2, (rows, cols))).astype(np.int8)
    w = oracle.pack_signs(s, "U")
    assert np.array_equal(oracle.unpack_rows(w, cols), s)
    # every bit past column `cols` is zero
    ld = w.shape[1]
    for c in range(cols, ld * 32):
        assert not ((w[:, c // 32] >> np.uint32(c % 32)) & 1).any()
    # an explicit, larger ld only adds zero words
    w2 = oracle.pack_signs(s, "U", ld_words=ld + 4)
    assert np.array_equal(w2[:, :ld], w) and not w2[:, ld:].any()


def test_bit_order_single_negative():
    """A single -1 at column c sets exactly bit c % 32 of word c // 32."""
    for c in (0, 1, 15, 16, 31, 32, 63, 64, 95):
        s = np.ones((1, 96), dtype=np.int8)
        s[0, c] = -1
        w = oracle.pack_signs(s, "U")
        expect = np.zeros(3, dtype=np.uint32)
        expect[c // 32] = np.uint32(1) << np.uint32(c % 32)
        assert np.array_equal(w[0], expect)
