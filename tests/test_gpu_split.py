"""lb_latent_forward and lb_expand_forward on the GPU against the fp64 oracle.

The latent is checked against oracle.latent; the expansion against
oracle.expand fed the GPU's own fp16 latent (so each half is judged alone);
the two in sequence against oracle.forward.  Token counts span the tcgen05
decode kernels (up to 32) and the prefill kernels (more), with ragged
shapes, a strided latent, null pointers in the half a call does not read,
and an integer-exact case compared bit for bit.
"""
import ctypes

import numpy as np
import pytest

import binarized_rank_linear_b200 as lb
import oracle
from binarized_rank_linear_b200 import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def oracle_paths(layer):
    return [dict(su=p["su"], sv=p["sv"], h=oracle.f16_to_f64(p["h"]), g=oracle.f16_to_f64(p["g"]),
                 l=oracle.f16_to_f64(p["l"])) for p in layer["paths"]]


def f16_to_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


CASES = [("tiny", 1), ("llama2_7b_q", 8), ("qwen3_14b_kv", 300)] + \
        [(None, m) for m in (1, 5, 32, 33, 257)]


@pytest.mark.parametrize("name,tokens", CASES)
def test_halves_against_the_oracle(name, tokens):
    layer = (synth.make_config(name, tokens) if name else
             synth.make_layer(384, 160, [64, 96], tokens, config_id=800))
    paths = gu.device_paths(layer)
    res = paths[1] if len(paths) > 1 else None
    x = gu.bf16_tensor(layer["x"])
    P = oracle_paths(layer)
    xo = oracle.bf16_bits_to_f64(layer["x"])

    z = lb.latent_forward(x, paths[0], res)
    zf = f16_to_f64(z)
    gu.assert_close(zf, oracle.latent(xo, P), f"latent {name} M={tokens}")

    y = lb.expand_forward(z, paths[0], res)
    gu.assert_close(gu.bf16_to_f64(y), oracle.expand(zf, P), f"expand {name} M={tokens}")
    gu.assert_close(gu.bf16_to_f64(y), oracle.forward(xo, P), f"both halves {name} M={tokens}")
    assert lb.device_status() == lb.LB_OK


@pytest.mark.parametrize("tokens", [7, 40, 300])
def test_strided_latent_and_unread_halves(tokens):
    """A latent with row stride r + 24 (the padding is never written), and
    each call given only the half of a path it reads (the rest null)."""
    import torch
    layer = synth.make_layer(256, 96, [32, 64], tokens, config_id=801)
    paths = gu.device_paths(layer)
    R = 96
    x = gu.bf16_tensor(layer["x"])
    zbuf = torch.full((tokens, R + 24), 7.0, dtype=torch.float16, device="cuda")
    y = torch.empty((tokens, 96), dtype=torch.bfloat16, device="cuda")

    def half(p, v_side):
        return lb.LbPath(0 if v_side else p.u_bits.data_ptr(), p.vt_bits.data_ptr() if v_side else 0,
                         0 if v_side else p.h.data_ptr(), p.g.data_ptr() if v_side else 0,
                         p.l.data_ptr() if v_side else 0, p.rank, 0, 0)

    L = lb.lib()
    mv, rv = half(paths[0], True), half(paths[1], True)
    assert L.lb_latent_forward(x.data_ptr(), tokens, 256, 256, ctypes.byref(mv), ctypes.byref(rv),
                               zbuf.data_ptr(), R + 24, None) == lb.LB_OK
    mu, ru = half(paths[0], False), half(paths[1], False)
    assert L.lb_expand_forward(zbuf.data_ptr(), tokens, 96, R + 24, ctypes.byref(mu), ctypes.byref(ru),
                               y.data_ptr(), 96, None) == lb.LB_OK
    torch.cuda.synchronize()
    assert bool((zbuf[:, R:] == 7.0).all())
    P = oracle_paths(layer)
    gu.assert_close(f16_to_f64(zbuf[:, :R]), oracle.latent(oracle.bf16_bits_to_f64(layer["x"]), P), "strided z")
    gu.assert_close(gu.bf16_to_f64(y), oracle.forward(oracle.bf16_bits_to_f64(layer["x"]), P), "strided y")


@pytest.mark.parametrize("tokens", [3, 32, 48])
def test_integer_exact_halves_are_bitwise(tokens):
    """Unit scales and x in {-1, 0, 1}: the latent and the output are small
    integers, exact in fp16 and bf16, so both halves equal the oracle exactly."""
    from tests.test_gpu_forward import integer_layer
    layer = integer_layer(512, 224, [64, 32], tokens, 100 + tokens)
    paths = gu.device_paths(layer)
    x = gu.bf16_tensor(layer["x"])
    z = lb.latent_forward(x, paths[0], paths[1])
    y = lb.expand_forward(z, paths[0], paths[1])
    P = oracle_paths(layer)
    xo = oracle.bf16_bits_to_f64(layer["x"])
    assert np.array_equal(f16_to_f64(z), oracle.latent(xo, P))
    assert np.array_equal(gu.bf16_to_f64(y), oracle.forward(xo, P))
