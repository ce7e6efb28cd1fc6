"""The seeded input generator: deterministic, right shapes and distributions."""
import numpy as np

from binarized_rank_linear_b200 import synth


def test_deterministic_and_seeded():
    a = synth.make_config("tiny")
    b = synth.make_config("tiny")
    c = synth.make_config("tiny", seed=1)
    assert np.array_equal(a["x"], b["x"])
    assert np.array_equal(a["paths"][0]["su"], b["paths"][0]["su"])
    assert not np.array_equal(a["x"], c["x"])


def test_shapes_and_values():
    d = synth.make_layer(96, 64, [32, 16], 5, config_id=77)
    assert d["x"].shape == (5, 96) and d["x"].dtype == np.uint16
    p0, p1 = d["paths"]
    assert p0["sv"].shape == (96, 32) and p0["su"].shape == (64, 32)
    assert p1["sv"].shape == (96, 16) and p1["l"].shape == (16,)
    for p in d["paths"]:
        assert set(np.unique(p["su"])) <= {-1, 1} and set(np.unique(p["sv"])) <= {-1, 1}
        for k in ("h", "g", "l"):
            assert p[k].dtype == np.float16 and (p[k] > 0).all()


def test_distributions():
    rng = synth.rng_for(0, 5, 0)
    x = synth.draw_x(rng, 64, 4096)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    assert abs(xf.mean()) < 0.01 and abs(xf.std() - 1) < 0.01
    s = synth.draw_signs(synth.rng_for(0, 5, 1), 512, 512)
    assert abs(s.mean()) < 0.01
    v = synth.draw_scale(synth.rng_for(0, 5, 2), 100000, "lognormal").astype(np.float64)
    assert abs(np.log(v).mean() + 3) < 0.01 and abs(np.log(v).std() - 0.5) < 0.01


def test_bf16_rounding_is_nearest_even():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5], dtype=np.float32)
    bits = synth.f32_to_bf16_bits(v)
    back = (bits.astype(np.uint32) << 16).view(np.float32)
    assert back.tolist() == [1.0, 1.0, 1.0 + 2 ** -6, -2.5]
