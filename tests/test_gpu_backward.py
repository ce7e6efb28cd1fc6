"""lb_linear_backward on the GPU against the fp64 oracle's backward pass.

Every gradient (dx, and per path dh, dg, dl) is compared element by element
with ``oracle.backward`` on the same seeded inputs, with the tolerances the
forward pass uses (relative L2 <= 5e-3, max error <= 1e-2 of the largest
magnitude), over token counts from 1 to 1000, ragged ranks (paths meeting
inside a 64-column K-block), one or two paths, and the Qwen3-14B linears at
1024 tokens.  Integer-exact inputs must give the oracle's scale gradients bit
for bit; a joint sign flip of latent pairs, CTA pairs against single-CTA
tiles, and repeated calls must give identical bits.  At the benchmark's 8192
tokens Euler's identity (sum_o h_o dh_o = <dy, y_p>, the same for g and l)
checks the scale gradients against forward calls.
"""
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


def draw_dy(tokens, n_out, seed):
    rng = np.random.default_rng(seed)
    return synth.f32_to_bf16_bits(rng.standard_normal((tokens, n_out), dtype=np.float32))


def run_backward(layer, dy_bits, paths=None, **kw):
    import torch
    paths = gu.device_paths(layer) if paths is None else paths
    x = gu.bf16_tensor(layer["x"])
    dy = gu.bf16_tensor(dy_bits)
    out = lb.linear_backward(x, dy, paths[0], paths[1] if len(paths) > 1 else None, **kw)
    torch.cuda.synchronize()
    assert lb.device_status() == lb.LB_OK
    return out


def host(out):
    dx = gu.bf16_to_f64(out["dx"]) if out["dx"] is not None else None
    return dx, out["dh"].double().cpu().numpy(), out["dg"].double().cpu().numpy(), \
        out["dl"].double().cpu().numpy()


def check_against_oracle(layer, dy_bits, out, what):
    ref = oracle.backward(oracle.bf16_bits_to_f64(layer["x"]), oracle.bf16_bits_to_f64(dy_bits), oracle_paths(layer))
    dx, dh, dg, dl = host(out)
    if dx is not None:
        gu.assert_close(dx, ref["dx"], f"{what} dx")
    offs = np.cumsum([0] + [len(v) for v in ref["dl"]])
    for j in range(len(ref["dh"])):
        gu.assert_close(dh[j], ref["dh"][j], f"{what} dh path {j}")
        gu.assert_close(dg[j], ref["dg"][j], f"{what} dg path {j}")
        gu.assert_close(dl[offs[j]:offs[j + 1]], ref["dl"][j], f"{what} dl path {j}")


CASES = [
    (256, 512, [64, 32], 1), (256, 512, [64, 32], 5), (256, 512, [64, 32], 37), (256, 512, [64, 32], 128),
    (256, 512, [64, 32], 129), (256, 512, [64, 32], 300), (512, 224, [96], 77),
    # paths meeting inside a 64-column K-block of the latent (r0 = 480), K not a multiple of 64
    (1056, 288, [480, 512], 200), (288, 1056, [480, 512], 1000),
    # many column tiles both ways
    (2048, 4096, [256, 224], 256),
]


@pytest.mark.parametrize("n_in,n_out,ranks,tokens", CASES)
def test_backward_against_oracle(n_in, n_out, ranks, tokens):
    layer = synth.make_layer(n_in, n_out, ranks, tokens, config_id=1400 + n_in + n_out + tokens)
    dy = draw_dy(tokens, n_out, 11 + tokens)
    check_against_oracle(layer, dy, run_backward(layer, dy), f"{n_in}x{n_out} r={ranks} M={tokens}")


@pytest.mark.parametrize("name,tokens", [("qwen3_14b_kv", 1024), ("qwen3_14b_qo", 512), ("qwen3_14b_gate", 1024),
                                         ("qwen3_14b_down", 512), ("llama2_7b_gate", 256)])
def test_backward_model_shapes(name, tokens):
    layer = synth.make_config(name, tokens)
    dy = draw_dy(tokens, layer["n_out"], 21)
    check_against_oracle(layer, dy, run_backward(layer, dy), f"{name} M={tokens}")


def test_backward_kv_at_full_size():
    """Qwen3-14B k/v at its full 8192 tokens, every output against the oracle:
    the launch plans of the benchmarked size (the weight-gradient products
    split over 9 token parts for dh, several for dg; 64 latent tiles)."""
    layer = synth.make_config("qwen3_14b_kv")
    M = layer["x"].shape[0]
    dy = draw_dy(M, layer["n_out"], 23)
    check_against_oracle(layer, dy, run_backward(layer, dy), f"qwen3_14b_kv M={M}")


def test_integer_exact_scale_gradients_are_bitwise():
    """Unit scales, x and dy in {-1, 0, 1}: every intermediate is a small
    integer, exact in fp16, bf16 and fp32, so dh, dg and dl match the oracle
    bit for bit (and dx too, where it stays within bf16's exact integers)."""
    rng = np.random.default_rng(31)
    n_in, n_out, ranks, tokens = 64, 96, [32, 64], 150
    layer = synth.make_layer(n_in, n_out, ranks, tokens, config_id=1450)
    for p in layer["paths"]:
        for k in ("h", "g", "l"):
            p[k] = np.ones_like(p[k])
    layer["x"] = synth.f32_to_bf16_bits(rng.integers(-1, 2, (tokens, n_in)).astype(np.float32))
    dy = synth.f32_to_bf16_bits((rng.integers(-1, 2, (tokens, n_out)) * (rng.random((tokens, n_out)) < 0.1))
                                .astype(np.float32))
    out = run_backward(layer, dy)
    ref = oracle.backward(oracle.bf16_bits_to_f64(layer["x"]), oracle.bf16_bits_to_f64(dy), oracle_paths(layer))
    dx, dh, dg, dl = host(out)
    assert np.array_equal(dh, np.stack(ref["dh"])) and np.array_equal(dg, np.stack(ref["dg"]))
    assert np.array_equal(dl, np.concatenate(ref["dl"]))
    exact = np.abs(ref["dx"]) <= 256
    assert np.array_equal(dx[exact], ref["dx"][exact])


def test_deterministic_sign_flip_invariant_and_pairs_agree():
    import torch
    n_in, n_out, ranks, tokens = 1024, 2048, [256, 224], 1100
    layer = synth.make_layer(n_in, n_out, ranks, tokens, config_id=1460)
    dy = draw_dy(tokens, n_out, 41)
    a = host(run_backward(layer, dy))
    b = host(run_backward(layer, dy))
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
    flipped = dict(layer, paths=[dict(p, su=p["su"] * np.where(np.arange(p["su"].shape[1]) % 3 == 0, -1, 1).astype(np.int8),
                                      sv=p["sv"] * np.where(np.arange(p["sv"].shape[1]) % 3 == 0, -1, 1).astype(np.int8))
                                 for p in layer["paths"]])
    c = host(run_backward(flipped, dy))
    for u, v in zip(a, c):
        assert np.array_equal(u, v)
    lb.set_prefill_pairs(False)
    try:
        d = host(run_backward(layer, dy))
    finally:
        lb.set_prefill_pairs(True)
    for u, v in zip(a, d):
        assert np.array_equal(u, v)
    torch.cuda.synchronize()


def test_without_dx_and_with_zero_tokens():
    import torch
    layer = synth.make_layer(256, 512, [64, 32], 40, config_id=1470)
    dy = draw_dy(40, 512, 51)
    full = host(run_backward(layer, dy))
    part = host(run_backward(layer, dy, want_dx=False))
    assert part[0] is None
    for u, v in zip(full[1:], part[1:]):
        assert np.array_equal(u, v)
    paths = gu.device_paths(layer)
    x0 = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    dy0 = torch.empty((0, 512), dtype=torch.bfloat16, device="cuda")
    out = lb.linear_backward(x0, dy0, paths[0], paths[1])
    torch.cuda.synchronize()
    assert all(bool((out[k] == 0).all()) for k in ("dh", "dg", "dl"))


def test_bad_arguments_write_nothing():
    import ctypes
    import torch
    layer = synth.make_layer(256, 128, [32], 8, config_id=1480)
    paths = gu.device_paths(layer)
    x = gu.bf16_tensor(layer["x"])
    dy = gu.bf16_tensor(draw_dy(8, 128, 3))
    dx = torch.full((8, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    dh = torch.full((1, 128), 7.0, device="cuda")
    dg = torch.full((1, 256), 7.0, device="cuda")
    dl = torch.full((32,), 7.0, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    c = paths[0].as_c()
    L = lb.lib()
    need = lb.backward_workspace_bytes(8, 256, 128, 32)
    bad = [dict(n_in=250), dict(ldx=100), dict(xp=x.data_ptr() + 2), dict(ws_bytes=need - 1), dict(dhp=None)]
    for b in bad:
        st = L.lb_linear_backward(b.get("xp", x.data_ptr()), dy.data_ptr(), 8, b.get("n_in", 256), 128,
                                  b.get("ldx", 256), 128, ctypes.byref(c), None, dx.data_ptr(), 256,
                                  b.get("dhp", dh.data_ptr()), dg.data_ptr(), dl.data_ptr(), ws.data_ptr(),
                                  b.get("ws_bytes", ws.numel()), None)
        assert st != lb.LB_OK, b
    torch.cuda.synchronize()
    for t in (dx, dh, dg, dl):
        assert bool((t == 7.0).all())
    assert lb.device_status() == lb.LB_OK


def test_euler_identity_at_benchmark_size():
    """Qwen3-14B gate/up at 8192 tokens: y is homogeneous of degree one in each
    scale vector of a path, so sum_o h_o dh_o, sum_i g_i dg_i and sum_k l_k dl_k
    all equal <dy, y_p>, y_p that path's own forward output (a separate
    lb_linear_forward call with the path alone).  dy is the layer's own output
    (normalised) plus unit noise: with a dy independent of y, <dy, y_p> is a
    sum of terms of random sign, orders of magnitude below the size of its
    terms, and its rounding error (bf16 operands) is not small against it."""
    import torch
    layer = synth.make_config("qwen3_14b_gate")
    M = layer["x"].shape[0]
    paths = gu.device_paths(layer)
    x = gu.bf16_tensor(layer["x"])
    y = lb.linear_forward(x, *paths).float()
    noise = torch.from_numpy(np.random.default_rng(61).standard_normal((M, layer["n_out"]), dtype=np.float32)).cuda()
    dy_t = (y / y.pow(2).mean().sqrt() + noise).to(torch.bfloat16)
    dy_bits = gu.bf16_bits(dy_t)
    out = run_backward(layer, dy_bits, paths=paths)
    dy = dy_t.double()
    dh, dg, dl = (out[k].double() for k in ("dh", "dg", "dl"))
    off = 0
    for j, p in enumerate(paths):
        yp = lb.linear_forward(x, p).double()
        lp = float((dy * yp).sum())
        for got in (float((p.h.double() * dh[j]).sum()), float((p.g.double() * dg[j]).sum()),
                    float((p.l.double() * dl[off:off + p.rank]).sum())):
            assert abs(got - lp) <= 5e-3 * abs(lp), (j, got, lp)
        off += p.rank
    assert torch.isfinite(out["dx"].float()).all()
