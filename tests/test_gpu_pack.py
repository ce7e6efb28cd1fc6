"""lb_pack_signs on the GPU against the oracle's own packer, bit for bit."""
import numpy as np
import pytest

import binarized_rank_linear_b200 as lb
import oracle
from tests.conftest import load_golden

pytestmark = pytest.mark.gpu


def torch():
    import torch as t
    return t


SPECIAL_F32 = np.array([0x00000000, 0x80000000, 0x80000001, 0x007fffff, 0x807fffff, 0x7fc00000,
                        0xffc00000, 0x7f800000, 0xff800000, 0x3f800000, 0xbf800000], dtype=np.uint32)


def random_source(rng, rows, cols, dtype):
    t = torch()
    if dtype == "i8":
        a = rng.integers(-128, 128, (rows, cols), dtype=np.int16).astype(np.int8)
        return a, t.from_numpy(a)
    f = rng.standard_normal((rows, cols)).astype(np.float32)
    # sprinkle special values: +-0, subnormals, NaNs, infinities
    mask = rng.random((rows, cols)) < 0.2
    f.view(np.uint32)[mask] = rng.choice(SPECIAL_F32, size=int(mask.sum()))
    if dtype == "f32":
        return f, t.from_numpy(f)
    if dtype == "f16":
        h = f.astype(np.float16)
        hb = h.view(np.uint16)
        m2 = rng.random((rows, cols)) < 0.05
        hb[m2] = rng.choice(np.array([0x8000, 0x8001, 0x7e00, 0xfe00, 0xfc00, 0x7c00], np.uint16), int(m2.sum()))
        return h, t.from_numpy(h)
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    m2 = rng.random((rows, cols)) < 0.05
    bits[m2] = rng.choice(np.array([0x8000, 0x8001, 0x7fc0, 0xffc0, 0xff80, 0x7f80], np.uint16), int(m2.sum()))
    return bits, t.from_numpy(bits.view(np.int16)).view(t.bfloat16)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16", "i8"])
@pytest.mark.parametrize("kind", ["U", "V"])
@pytest.mark.parametrize("rows,cols", [(1, 1), (7, 33), (64, 288), (300, 96), (33, 1000)])
def test_pack_matches_oracle(dtype, kind, rows, cols):
    rng = np.random.default_rng(rows * 7919 + cols)
    host, src = random_source(rng, rows, cols, dtype)
    got = lb.pack_signs(src.cuda(), kind).cpu().numpy().view(np.uint32)
    expect = oracle.pack_signs(host, kind, dtype)
    assert got.shape == expect.shape
    assert np.array_equal(got, expect)


@pytest.mark.parametrize("kind", ["U", "V"])
def test_padding_words_are_written_zero(kind):
    t = torch()
    rng = np.random.default_rng(5)
    s = (1 - 2 * rng.integers(0, 2, (40, 70))).astype(np.int8)
    packed_cols = 70 if kind == "U" else 40
    ld = oracle.packed_ld_words(packed_cols) + 5
    rows = 40 if kind == "U" else 70
    dst = t.full((rows, ld), -1, dtype=t.int32, device="cuda")
    st = lb.lib().lb_pack_signs(t.from_numpy(s).cuda().data_ptr(), lb.LB_I8,
                                lb.LB_FACTOR_U if kind == "U" else lb.LB_FACTOR_V, 40, 70, 70,
                                dst.data_ptr(), ld, None)
    assert st == lb.LB_OK
    t.cuda.synchronize()
    got = dst.cpu().numpy().view(np.uint32)
    assert np.array_equal(got, oracle.pack_signs(s, kind, "i8", ld_words=ld))


def test_hand_packed_fixture():
    fx = load_golden("pack_hand.txt")
    t = torch()
    u = np.ones((fx["u_rows"], fx["u_cols"]), dtype=np.int8)
    for row, cols in enumerate(fx["u_negative_columns"]):
        u[row, cols] = -1
    got_u = lb.pack_signs(t.from_numpy(u).cuda(), "U", ld_words=4).cpu().numpy().view(np.uint32)
    got_v = lb.pack_signs(t.from_numpy(u.T.copy()).cuda(), "V", ld_words=4).cpu().numpy().view(np.uint32)
    assert np.array_equal(got_u, np.array(fx["u_words"], np.uint32))
    assert np.array_equal(got_v, np.array(fx["v_words"], np.uint32))
    sp = np.array(fx["special_f32_bits"], np.uint32).view(np.float32)[None, :]
    w = lb.pack_signs(t.from_numpy(sp.copy()).cuda(), "U").cpu().numpy().view(np.uint32)
    assert int(w[0, 0]) == fx["special_word0"]


def test_strided_source():
    t = torch()
    rng = np.random.default_rng(11)
    big = rng.standard_normal((50, 100)).astype(np.float32)
    src = t.from_numpy(big).cuda()[:, 10:77]          # row stride 100, 67 columns
    got = lb.pack_signs(src, "U").cpu().numpy().view(np.uint32)
    assert np.array_equal(got, oracle.pack_signs(big[:, 10:77], "U", "f32"))
    got_v = lb.pack_signs(src, "V").cpu().numpy().view(np.uint32)
    assert np.array_equal(got_v, oracle.pack_signs(big[:, 10:77], "V", "f32"))
