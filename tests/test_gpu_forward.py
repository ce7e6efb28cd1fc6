"""lb_linear_forward on the GPU against the fp64 oracle.

Every workload of the synthetic table runs at each of its token counts; the
prefill workloads (8192 tokens) are checked on a sample of token rows that
the oracle computes one by one.  Edge cases: the token sweep around the
decode/prefill boundary, ragged shapes with r1 != r2, an integer-exact case
that must match bit for bit, sign-flip invariance (bitwise), determinism,
workspace contents, strided outputs and canaries, and the status word.
"""
import numpy as np
import pytest

import binarized_rank_linear_b200 as lb
import oracle
from binarized_rank_linear_b200 import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def torch():
    import torch as t
    return t


DECODE_CASES = [(name, m) for name, c in sorted(synth.CONFIGS.items()) if c.tokens[0] <= 32
                for m in c.tokens]


@pytest.mark.parametrize("name,tokens", DECODE_CASES)
def test_decode_configs(name, tokens):
    layer = synth.make_config(name, tokens)
    y = gu.bf16_to_f64(gu.run_gpu(layer))
    gu.assert_close(y, gu.oracle_y(layer), f"{name} M={tokens}")


PREFILL = [name for name, c in sorted(synth.CONFIGS.items()) if c.tokens[0] > 32]


@pytest.mark.parametrize("name", PREFILL)
def test_prefill_configs_every_row(name):
    """The Qwen3-14B linears at 8192 tokens, in the launch configuration the
    benchmark times (CTA pairs where the tile plan takes them), checked whole:
    every output against the fp64 oracle (about 30 s of oracle time for
    gate/up or down on a 16-core host).  Besides the whole-matrix criteria,
    every 128-row block must meet the relative L2 bound on its own, so a fault
    confined to one tile of the persistent schedule cannot hide in the
    average."""
    layer = synth.make_config(name)
    M = layer["x"].shape[0]
    y = gu.bf16_to_f64(gu.run_gpu(layer))
    assert np.all(np.isfinite(y))
    ref = gu.oracle_y(layer)
    gu.assert_close(y, ref, f"{name} all {M} rows")
    for r0 in range(0, M, 128):
        d = np.linalg.norm(y[r0:r0 + 128] - ref[r0:r0 + 128]) / np.linalg.norm(ref[r0:r0 + 128])
        assert d <= gu.REL_L2_TOL, f"{name} rows {r0}..{r0 + 127}: relative L2 {d:.3e}"


@pytest.mark.parametrize("tokens", [1, 2, 7, 8, 9, 16, 17, 31, 32, 33, 64, 255, 256, 257])
def test_token_sweep_ragged_shape(tokens):
    layer = synth.make_layer(384, 160, [64, 96], tokens, config_id=500)
    y = gu.bf16_to_f64(gu.run_gpu(layer))
    gu.assert_close(y, gu.oracle_y(layer), f"M={tokens}")


@pytest.mark.parametrize("n_in,n_out,ranks", [(256, 5120, [64, 32]), (64, 32, [2432, 2432])])
def test_prefill_tile_shapes_ragged(n_in, n_out, ranks):
    """1000 tokens over many output tiles: 1000 = 7 x 128 + 104 leaves the
    last row tile partly outside the batch, and a latent of 96 (first case)
    is one and a half K-blocks; the second case has a 4864-wide latent, so
    contraction 1 runs more tiles than there are SMs."""
    layer = synth.make_layer(n_in, n_out, ranks, 1000, config_id=700 + n_out)
    y = gu.bf16_to_f64(gu.run_gpu(layer))
    gu.assert_close(y, gu.oracle_y(layer), f"{n_in}x{n_out} r={ranks} M=1000")


# Shapes whose contractions take each family of the prefill kernel's tile
# plans on a 148-SM B200 (128-row tiles of width 32 .. 256, one or two waves;
# 256-row tiles at 2100 tokens), each checked whole against the oracle.  The
# plan is the library's choice; the ids record which one each shape took when
# the cases were picked.
# Shapes whose planned tiles cover the kernel's variants (ids: the contraction
# and its plan; "pair" = CTA pairs sharing each MMA, "h2" = two 128-row halves
# per CTA).
TILE_PLAN_CASES = [
    pytest.param(129, 256, 256, [32, 32], id="m129-c1-w32"),
    pytest.param(129, 256, 4096, [32, 32], id="m129-c2-w64"),
    pytest.param(520, 256, 2048, [32, 32], id="m520-c2-w96"),
    pytest.param(1000, 256, 2048, [32, 32], id="m1000-c2-w128"),
    pytest.param(700, 256, 4096, [32, 32], id="m700-c2-pair-w192"),
    pytest.param(2600, 256, 2048, [32, 32], id="m2600-c2-pair-w160-2waves"),
    pytest.param(2100, 256, 4096, [160, 160], id="m2100-c2-pair-w256"),
    pytest.param(2600, 256, 256, [512, 512], id="m2600-c1-pair-w192"),
    pytest.param(3000, 256, 416, [512, 512], id="m3000-c1-pair-w192-ragged-m"),
    pytest.param(900, 512, 6016, [256, 224], id="m900-c2-pair-w192-ragged-n"),
    pytest.param(520, 256, 8192, [512, 512], id="m520-c2-pair-h2-w224-ragged"),
    pytest.param(5000, 1024, 256, [512, 512], id="m5000-c1-pair-h2-w160-ragged"),
    # K not a multiple of the 64-column K-block in both contractions, and the
    # two paths meeting inside a K-block of contraction 2 (r0 = 480)
    pytest.param(5000, 1056, 288, [480, 512], id="m5000-c1-pair-h2-ragged-k"),
    pytest.param(520, 288, 8192, [480, 512], id="m520-c2-pair-h2-ragged-k-mid-block-paths"),
    pytest.param(3000, 1056, 2048, [480, 512], id="m3000-pair-both-ragged-k"),
    # few tiles of a long K in contraction 1 (the Qwen3-14B k/v shape at fewer tokens)
    pytest.param(2048, 5120, 1024, [224, 224], id="m2048-c1-few-tiles-long-k"),
    pytest.param(1000, 4096, 512, [128, 96], id="m1000-c1-long-k-ragged-m"),
    pytest.param(700, 2048, 256, [32, 32], id="m700-c1-narrow-long-k"),
]


@pytest.fixture(params=[True, False], ids=["pairs", "single-cta"])
def prefill_pairs(request):
    """Runs a test with CTA-pair prefill tiles allowed (the default) and with
    single-CTA tiles only (lb_set_prefill_pairs), restoring the default."""
    lb.set_prefill_pairs(request.param)
    yield request.param
    lb.set_prefill_pairs(True)


@pytest.mark.parametrize("tokens,n_in,n_out,ranks", TILE_PLAN_CASES)
def test_prefill_tile_plans(tokens, n_in, n_out, ranks, prefill_pairs):
    layer = synth.make_layer(n_in, n_out, ranks, tokens, config_id=900 + n_out + sum(ranks))
    y = gu.bf16_to_f64(gu.run_gpu(layer))
    gu.assert_close(y, gu.oracle_y(layer), f"{n_in}x{n_out} r={ranks} M={tokens} pairs={prefill_pairs}")


@pytest.mark.parametrize("n_in,n_out,ranks", [(32, 32, [32]), (96, 64, [32]), (64, 800, [32, 64]),
                                              (1056, 224, [160, 32]), (4096, 96, [288])])
def test_small_and_asymmetric_shapes(n_in, n_out, ranks):
    for tokens in (1, 5, 40):
        layer = synth.make_layer(n_in, n_out, ranks, tokens, config_id=600 + n_in + n_out)
        y = gu.bf16_to_f64(gu.run_gpu(layer))
        gu.assert_close(y, gu.oracle_y(layer), f"{n_in}x{n_out} r={ranks} M={tokens}")


def integer_layer(n_in, n_out, ranks, tokens, seed, zero_frac=0.9):
    rng = np.random.default_rng(seed)
    paths = []
    for r in ranks:
        paths.append(dict(sv=(1 - 2 * rng.integers(0, 2, (n_in, r))).astype(np.int8),
                          su=(1 - 2 * rng.integers(0, 2, (n_out, r))).astype(np.int8),
                          h=np.ones(n_out, np.float16), g=np.ones(n_in, np.float16),
                          l=np.ones(r, np.float16)))
    xf = rng.integers(-1, 2, (tokens, n_in)).astype(np.float32)
    xf[rng.random((tokens, n_in)) < zero_frac] = 0.0  # keep |y| small
    x = (xf.view(np.uint32) >> 16).astype(np.uint16)
    return dict(x=x, paths=paths, n_in=n_in, n_out=n_out)


def bf16_rne(v: np.ndarray) -> np.ndarray:
    return synth.f32_to_bf16_bits(v.astype(np.float32))


@pytest.mark.parametrize("tokens", [1, 3, 8, 32, 40, 129, 300, 1000])
def test_integer_exact_is_bitwise(tokens):
    """Unit scales and x in {-1, 0, 1}: every intermediate is a small integer,
    exact in fp16, bf16 and fp32, so the GPU must equal the oracle (rounded
    to bf16) bit for bit.  Pins sign orientation, pack layout and transposes."""
    # sparser x for the larger batches keeps every |y| within 256
    layer = integer_layer(512, 224, [64, 32], tokens, tokens, 0.9 if tokens < 100 else 0.97)
    ref = gu.oracle_y(layer)
    assert np.abs(ref).max() <= 256 and np.array_equal(ref, np.rint(ref))
    got = gu.bf16_bits(gu.run_gpu(layer))
    assert np.array_equal(got, bf16_rne(ref))


@pytest.mark.parametrize("n_in,n_out,ranks,tokens", [(256, 8192, [512, 512], 520), (256, 256, [512, 512], 2600),
                                                     (512, 224, [64, 32], 300), (512, 224, [64, 32], 1000),
                                                     (288, 8192, [480, 512], 520), (4096, 256, [128, 96], 1000)],
                         ids=["c2-h2", "c1-wide", "m300", "m1000", "ragged-k", "c1-long-k"])
def test_integer_exact_prefill_tiles_are_bitwise(n_in, n_out, ranks, tokens, prefill_pairs):
    """The integer-exact case on prefill shapes, on CTA pairs and on single
    CTAs.  Every value is an integer well inside fp32's exact range and z
    inside fp16's, so the GPU equals the oracle rounded to bf16 (round to
    nearest even) bit for bit."""
    layer = integer_layer(n_in, n_out, ranks, tokens, 31 + tokens, 0.95)
    ref = gu.oracle_y(layer)
    assert np.abs(ref).max() < 2 ** 24 and np.array_equal(ref, np.rint(ref))
    got = gu.bf16_bits(gu.run_gpu(layer))
    assert np.array_equal(got, bf16_rne(ref))


@pytest.mark.parametrize("tokens,n_in,n_out,ranks", [(700, 256, 4096, [32, 32]), (2100, 256, 4096, [160, 160]),
                                                     (520, 256, 8192, [512, 512]), (2048, 5120, 1024, [224, 224])])
def test_pair_and_single_cta_tiles_agree_bitwise(tokens, n_in, n_out, ranks):
    """Every output element sums the same K-steps in the same order whether
    its row sits in a single-CTA tile or in a CTA pair's, and the epilogue
    rounds it the same way, so the two give the same bits."""
    layer = synth.make_layer(n_in, n_out, ranks, tokens, config_id=1900 + n_out + sum(ranks))
    paths = gu.device_paths(layer)
    try:
        lb.set_prefill_pairs(True)
        a = gu.bf16_bits(gu.run_gpu(layer, paths=paths))
        lb.set_prefill_pairs(False)
        b = gu.bf16_bits(gu.run_gpu(layer, paths=paths))
    finally:
        lb.set_prefill_pairs(True)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("tokens", [1, 8, 300])
def test_sign_flip_invariance_is_bitwise(tokens):
    layer = synth.make_layer(1024, 512, [96, 64], tokens, config_id=700)
    y0 = gu.bf16_bits(gu.run_gpu(layer))
    rng = np.random.default_rng(2)
    for p in layer["paths"]:
        cols = rng.random(p["su"].shape[1]) < 0.5
        p["su"] = np.where(cols[None, :], -p["su"], p["su"]).astype(np.int8)
        p["sv"] = np.where(cols[None, :], -p["sv"], p["sv"]).astype(np.int8)
    y1 = gu.bf16_bits(gu.run_gpu(layer))
    assert np.array_equal(y0, y1)


@pytest.mark.parametrize("tokens", [1, 16, 300])
def test_deterministic_and_workspace_independent(tokens):
    """Repeated calls give the same bits whatever the workspace held before
    (CUDA-core, tcgen05 decode and prefill pair kernels)."""
    t = torch()
    layer = synth.make_config("llama2_7b_gate", tokens)
    paths = gu.device_paths(layer)
    x = gu.bf16_tensor(layer["x"])
    c = synth.CONFIGS["llama2_7b_gate"]
    need = lb.forward_workspace_bytes(tokens, c.n_in, c.n_out, c.rank, c.rank)
    outs = []
    for fill in (0, 0xFF, 0x7C):
        ws = t.full((need,), fill, dtype=t.uint8, device="cuda")
        outs.append(gu.bf16_bits(lb.linear_forward(x, paths[0], paths[1], workspace=ws)))
    assert all(np.array_equal(outs[0], o) for o in outs[1:])


@pytest.mark.parametrize("tokens", [2, 5, 300, 1000])
def test_strided_io_and_canaries(tokens, prefill_pairs):
    """x and y with row strides past their widths, on every kernel family
    (the prefill ones on CTA pairs and on single CTAs): y right, and nothing
    written past its columns or rows."""
    t = torch()
    layer = synth.make_layer(256, 128, [32, 64], tokens, config_id=800)
    paths = gu.device_paths(layer)
    xb = t.zeros((tokens, 264), dtype=t.bfloat16, device="cuda")
    xb[:, :256] = gu.bf16_tensor(layer["x"])
    ybig = t.full((tokens + 2, 136), 12345.0, dtype=t.bfloat16, device="cuda")
    y = ybig[:tokens, :128]
    lb.linear_forward(xb[:, :256], paths[0], paths[1], y=y)
    t.cuda.synchronize()
    gu.assert_close(gu.bf16_to_f64(y.contiguous()), gu.oracle_y(layer), f"strided M={tokens}")
    assert bool((ybig[:, 128:] == 12345.0).all()) and bool((ybig[tokens:] == 12345.0).all())


def test_bad_arguments_write_nothing():
    t = torch()
    layer = synth.make_layer(256, 128, [32], 3, config_id=801)
    paths = gu.device_paths(layer)
    x = gu.bf16_tensor(layer["x"])
    y = t.full((3, 128), 7.0, dtype=t.bfloat16, device="cuda")
    ws = t.empty(1 << 20, dtype=t.uint8, device="cuda")
    c = paths[0].as_c()
    L = lb.lib()
    import ctypes
    for args in [(x.data_ptr(), 3, 250, 128, 256), (x.data_ptr() + 2, 3, 256, 128, 256),
                 (x.data_ptr(), 3, 256, 128, 100)]:
        st = L.lb_linear_forward(*args, ctypes.byref(c), None, y.data_ptr(), 128, ws.data_ptr(),
                                 ws.numel(), None)
        assert st != lb.LB_OK
    st = L.lb_linear_forward(x.data_ptr(), 3, 256, 128, 256, ctypes.byref(c), None, y.data_ptr(), 128,
                             ws.data_ptr(), 16, None)
    assert st == lb.LB_ERR_WORKSPACE_TOO_SMALL
    t.cuda.synchronize()
    assert bool((y == 7.0).all())
    assert lb.device_status() == lb.LB_OK


def test_zero_tokens_is_a_noop():
    t = torch()
    layer = synth.make_layer(256, 128, [32], 1, config_id=802)
    paths = gu.device_paths(layer)
    x = t.empty((0, 256), dtype=t.bfloat16, device="cuda")
    y = lb.linear_forward(x, paths[0])
    assert y.shape == (0, 128)


def test_range_overflow_sets_status_not_fault():
    """g (.) x beyond the fp16 range on the tensor-core decode path (5..32
    tokens) raises LB_ERR_RANGE on the status word (the kernels keep running;
    nothing faults)."""
    layer = synth.make_layer(256, 128, [32], 8, config_id=803)
    big = np.full((8, 256), 1e8, dtype=np.float32)
    layer["x"] = synth.f32_to_bf16_bits(big)
    assert lb.device_status() == lb.LB_OK
    gu.run_gpu(layer)
    assert lb.device_status() == lb.LB_ERR_RANGE
    assert lb.device_status() == lb.LB_OK          # read clears it


def test_small_batch_path_is_fp32_throughout():
    """1..4 tokens run in fp32 up to the bf16 output: inputs far beyond the
    fp16 range are fine there."""
    layer = synth.make_layer(256, 128, [32, 64], 3, config_id=804)
    xf = oracle.bf16_bits_to_f64(layer["x"]) * 2.0 ** 40
    layer["x"] = synth.f32_to_bf16_bits(xf.astype(np.float32))
    y = gu.bf16_to_f64(gu.run_gpu(layer))
    gu.assert_close(y, gu.oracle_y(layer), "x * 2^40")
    assert lb.device_status() == lb.LB_OK


def test_non_default_stream():
    t = torch()
    layer = synth.make_config("llama2_7b_q", 8)
    paths = gu.device_paths(layer)
    x = gu.bf16_tensor(layer["x"])
    s = t.cuda.Stream()
    with t.cuda.stream(s):
        y = lb.linear_forward(x, paths[0], paths[1], stream=s)
    s.synchronize()
    gu.assert_close(gu.bf16_to_f64(y), gu.oracle_y(layer), "side stream")


def test_layer_object():
    layer = synth.make_config("tiny")
    mod = lb.LittleBitLinear.from_factors(layer["paths"])
    y = mod(gu.bf16_tensor(layer["x"]))
    gu.assert_close(gu.bf16_to_f64(y), gu.oracle_y(layer), "module")


@pytest.mark.parametrize("tokens", [1, 3, 4, 5, 37, 128])
def test_host_call_on_pinned_buffers_writes_y_in_place(tokens):
    """1-128 tokens on pinned host buffers: x reaches x_dev through the gather
    kernel and the last kernel writes y to host memory directly, so y_dev
    keeps its sentinel, x_dev holds x, and y_host has the device call's bits."""
    import torch
    layer = synth.make_layer(512, 224, [64, 32], tokens, config_id=881)
    paths = gu.device_paths(layer)
    x = gu.bf16_tensor(layer["x"])
    ref = lb.linear_forward(x, paths[0], paths[1])
    x_host = x.cpu().pin_memory()
    y_host = torch.full((tokens, 224), 3.0, dtype=torch.bfloat16).pin_memory()
    x_dev = torch.full_like(x, 5.0)
    y_dev = torch.full((tokens, 224), 7.0, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(16, lb.forward_workspace_bytes(tokens, 512, 224, 64, 32)), dtype=torch.uint8, device="cuda")
    lb.linear_forward_host(x_host, paths[0], paths[1], y_host, x_dev, y_dev, ws)
    torch.cuda.synchronize()
    assert lb.device_status() == lb.LB_OK
    assert np.array_equal(gu.bf16_bits(y_host), gu.bf16_bits(ref))
    assert np.array_equal(gu.bf16_bits(x_dev), gu.bf16_bits(x)) and bool((y_dev == 7.0).all())


@pytest.mark.parametrize("tokens", [1, 37])
def test_back_to_back_host_calls_share_device_buffers(tokens):
    """Several host-buffer calls queued on one stream without a sync, all
    through the same x_dev: each call's gather kernel must wait for the
    previous call's kernels before it overwrites x_dev, so every y_host holds
    its own input's result."""
    import torch
    layers = [synth.make_layer(512, 224, [64, 32], tokens, config_id=890 + i) for i in range(4)]
    paths = gu.device_paths(layers[0])
    x_dev = torch.empty((tokens, 512), dtype=torch.bfloat16, device="cuda")
    y_dev = torch.empty((tokens, 224), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(16, lb.forward_workspace_bytes(tokens, 512, 224, 64, 32)), dtype=torch.uint8, device="cuda")
    xs = [gu.bf16_tensor(L["x"]).cpu().pin_memory() for L in layers]
    ys = [torch.zeros((tokens, 224), dtype=torch.bfloat16).pin_memory() for _ in layers]
    torch.cuda.synchronize()
    for _ in range(3):
        for xh, yh in zip(xs, ys):
            lb.linear_forward_host(xh, paths[0], paths[1], yh, x_dev, y_dev, ws)
    torch.cuda.synchronize()
    assert lb.device_status() == lb.LB_OK
    for xh, yh in zip(xs, ys):
        ref = lb.linear_forward(xh.cuda(), paths[0], paths[1])
        assert np.array_equal(gu.bf16_bits(yh), gu.bf16_bits(ref))


def test_host_call_on_pageable_buffers_copies():
    """Pageable host memory is not visible to the kernels: the call copies x
    into x_dev and y out of y_dev, with the same bits."""
    import torch
    tokens = 2
    layer = synth.make_layer(512, 224, [64, 32], tokens, config_id=882)
    paths = gu.device_paths(layer)
    x = gu.bf16_tensor(layer["x"])
    ref = lb.linear_forward(x, paths[0], paths[1])
    x_host = x.cpu().clone()
    y_host = torch.full((tokens, 224), 3.0, dtype=torch.bfloat16)
    assert not x_host.is_pinned() and not y_host.is_pinned()
    x_dev = torch.full_like(x, 5.0)
    y_dev = torch.full((tokens, 224), 7.0, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(16, lb.forward_workspace_bytes(tokens, 512, 224, 64, 32)), dtype=torch.uint8, device="cuda")
    lb.linear_forward_host(x_host, paths[0], paths[1], y_host, x_dev, y_dev, ws)
    torch.cuda.synchronize()
    assert lb.device_status() == lb.LB_OK
    assert np.array_equal(gu.bf16_bits(y_host), gu.bf16_bits(ref))
    assert np.array_equal(gu.bf16_bits(x_dev), gu.bf16_bits(x)) and np.array_equal(gu.bf16_bits(y_dev), gu.bf16_bits(ref))


@pytest.mark.parametrize("tokens", [1, 8, 300])
def test_host_buffer_call_equals_device_call(tokens):
    """lb_linear_forward_host: x from pinned host memory and y back to it,
    through the caller's device buffers; the same kernels as the device call,
    so the same bits."""
    import torch
    layer = synth.make_layer(512, 224, [64, 32], tokens, config_id=880)
    paths = gu.device_paths(layer)
    res = paths[1] if len(paths) > 1 else None
    x = gu.bf16_tensor(layer["x"])
    ref = lb.linear_forward(x, paths[0], res)
    x_host = x.cpu().pin_memory()
    y_host = torch.full((tokens, 224), 3.0, dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)
    y_dev = torch.empty((tokens, 224), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(16, lb.forward_workspace_bytes(tokens, 512, 224, 64, 32)), dtype=torch.uint8, device="cuda")
    lb.linear_forward_host(x_host, paths[0], res, y_host, x_dev, y_dev, ws)
    torch.cuda.synchronize()
    assert lb.device_status() == lb.LB_OK
    assert np.array_equal(gu.bf16_bits(y_host), gu.bf16_bits(ref))
    gu.assert_close(gu.bf16_to_f64(y_host), gu.oracle_y(layer), f"host buffers M={tokens}")


@pytest.mark.parametrize("tokens", [1, 3, 37])
def test_chained_host_calls_read_the_previous_output(tokens):
    """Host-buffer calls chained layer to layer on one stream without a sync:
    the y_host of one call is the x_host of the next.  Each call's gather
    kernel must read x_host only after the previous call's last kernel has
    stored it (that kernel releases its dependents before its stores), so the
    chain gives the bits of the same chain run through device buffers."""
    import torch
    n = 512
    layer = synth.make_layer(n, n, [64, 32], tokens, config_id=883)
    paths = gu.device_paths(layer)
    x = gu.bf16_tensor(layer["x"])
    ws = torch.empty(max(16, lb.forward_workspace_bytes(tokens, n, n, 64, 32)), dtype=torch.uint8, device="cuda")
    depth = 5
    # the reference chain: device buffers, synchronised after every call
    refs, cur = [], x
    for _ in range(depth):
        cur = lb.linear_forward(cur, paths[0], paths[1], workspace=ws)
        torch.cuda.synchronize()
        refs.append(cur.clone())
    hosts = [x.cpu().pin_memory()] + [torch.full((tokens, n), 3.0, dtype=torch.bfloat16).pin_memory()
                                      for _ in range(depth)]
    x_dev = torch.empty_like(x)
    y_dev = torch.empty((tokens, n), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    for d in range(depth):
        lb.linear_forward_host(hosts[d], paths[0], paths[1], hosts[d + 1], x_dev, y_dev, ws)
    torch.cuda.synchronize()
    assert lb.device_status() == lb.LB_OK
    for d in range(depth):
        assert np.array_equal(gu.bf16_bits(hosts[d + 1]), gu.bf16_bits(refs[d])), f"layer {d}"
    gu.assert_close(gu.bf16_to_f64(hosts[1]), gu.oracle_y(layer), f"first layer M={tokens}")


def test_few_tiles_long_k_is_deterministic_and_sign_flip_invariant():
    """The Qwen3-14B k/v shape at 2048 tokens (few output tiles, a long K):
    repeated calls give the same bits, and so does a joint sign flip of latent
    pairs."""
    layer = synth.make_layer(5120, 1024, [224, 224], 2048, config_id=1600)
    paths = gu.device_paths(layer)
    y0 = gu.bf16_bits(gu.run_gpu(layer, paths=paths))
    for _ in range(3):
        assert np.array_equal(gu.bf16_bits(gu.run_gpu(layer, paths=paths)), y0)
    flip = lambda a: (a * np.where(np.arange(a.shape[1]) % 2 == 0, -1, 1)).astype(np.int8)
    flipped = dict(layer, paths=[dict(p, su=flip(p["su"]), sv=flip(p["sv"])) for p in layer["paths"]])
    assert np.array_equal(gu.bf16_bits(gu.run_gpu(flipped)), y0)
    gu.assert_close(oracle.bf16_bits_to_f64(y0), gu.oracle_y(layer), "k/v shape, 2048 tokens")
