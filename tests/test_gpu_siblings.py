"""lb_linear_forward_siblings on the GPU: every projection of a group that
shares x against the fp64 oracle on that projection alone.

Up to 128 tokens the whole group runs as one launch pair (the latents of all
the group's paths side by side, the output rows of all its projections in one
grid): CUDA-core kernels for 1..4 tokens, tcgen05 kernels for 5..128; more
tokens run each projection's own launches.  Cases: a Qwen3-14B
attention group (q with a 5120-wide output and k, v with 1024, different
ranks), a Llama-2-7B gate/up pair, ragged small groups that mix projections
with and without the residual path, an integer-exact group compared bit for
bit, and the per-layer fallback compared bit for bit with separate calls.
"""
import numpy as np
import pytest

import binarized_rank_linear_b200 as lb
from binarized_rank_linear_b200 import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def group_layers(specs, n_in, tokens, seed):
    """specs: [(n_out, ranks)]; the layers share one x."""
    layers = [synth.make_layer(n_in, n_out, ranks, tokens, config_id=seed + j) for j, (n_out, ranks) in
              enumerate(specs)]
    for lay in layers[1:]:
        lay["x"] = layers[0]["x"]
    return layers


def config_group(names, tokens):
    layers = [synth.make_config(n, tokens, seed=j) for j, n in enumerate(names)]
    for lay in layers[1:]:
        lay["x"] = layers[0]["x"]
    return layers


def run_group(layers):
    import torch
    x = gu.bf16_tensor(layers[0]["x"])
    dev = [gu.device_paths(lay) for lay in layers]
    ys = lb.linear_forward_siblings(x, [(p[0], p[1] if len(p) > 1 else None) for p in dev])
    torch.cuda.synchronize()
    assert lb.device_status() == lb.LB_OK
    return ys, dev, x


@pytest.mark.parametrize("tokens", [1, 2, 3, 4, 5, 40, 64, 128, 129])
def test_qwen3_attention_group(tokens):
    layers = config_group(["qwen3_14b_qo", "qwen3_14b_kv", "qwen3_14b_kv"], tokens)
    ys, _, _ = run_group(layers)
    for j, (lay, y) in enumerate(zip(layers, ys)):
        gu.assert_close(gu.bf16_to_f64(y), gu.oracle_y(lay), f"projection {j} M={tokens}")


@pytest.mark.parametrize("tokens", [1, 4, 16, 100])
def test_llama2_gate_up_pair(tokens):
    layers = config_group(["llama2_7b_gate", "llama2_7b_gate"], tokens)
    ys, _, _ = run_group(layers)
    for j, (lay, y) in enumerate(zip(layers, ys)):
        gu.assert_close(gu.bf16_to_f64(y), gu.oracle_y(lay), f"projection {j} M={tokens}")


SMALL_GROUPS = [
    [(96, [64]), (160, [32, 64]), (64, [96, 32]), (32, [32])],  # four projections, mixed paths
    [(512, [32, 32])],                                            # a group of one
    [(256, [128]), (256, [128])],
]


@pytest.mark.parametrize("specs", SMALL_GROUPS)
@pytest.mark.parametrize("tokens", [1, 3, 4, 5, 33, 300])
def test_ragged_groups(specs, tokens):
    layers = group_layers(specs, 256, tokens, 950 + 10 * len(specs))
    ys, _, _ = run_group(layers)
    for j, (lay, y) in enumerate(zip(layers, ys)):
        assert y.shape == (tokens, specs[j][0])
        gu.assert_close(gu.bf16_to_f64(y), gu.oracle_y(lay), f"{specs} projection {j} M={tokens}")


@pytest.mark.parametrize("tokens", [1, 4, 8, 100])
def test_integer_exact_group_is_bitwise(tokens):
    from tests.test_gpu_forward import bf16_rne, integer_layer
    # sparser x for the larger batches keeps every |y| within 256
    layers = [integer_layer(512, n_out, ranks, tokens, 300 + j, 0.9 if tokens < 50 else 0.97)
              for j, (n_out, ranks) in enumerate([(224, [64, 32]), (96, [32]), (128, [64, 64])])]
    for lay in layers[1:]:
        lay["x"] = layers[0]["x"]
    ys, _, _ = run_group(layers)
    for lay, y in zip(layers, ys):
        ref = gu.oracle_y(lay)
        assert np.abs(ref).max() <= 256 and np.array_equal(ref, np.rint(ref))
        assert np.array_equal(gu.bf16_bits(y), bf16_rne(ref))


@pytest.mark.parametrize("tokens", [129, 300])
def test_more_tokens_equal_separate_calls_bitwise(tokens):
    """Past 128 tokens each projection runs its own launches: the outputs are
    those of separate lb_linear_forward calls, bit for bit."""
    layers = group_layers([(160, [32, 64]), (64, [96])], 256, tokens, 990)
    ys, dev, x = run_group(layers)
    for y, p in zip(ys, dev):
        ref = lb.linear_forward(x, p[0], p[1] if len(p) > 1 else None)
        assert np.array_equal(gu.bf16_bits(y), gu.bf16_bits(ref))


def test_outputs_outside_the_rows_are_untouched():
    """Strided outputs: the padding columns of every projection's y keep their
    canary values."""
    import torch
    layers = group_layers([(96, [64]), (64, [32, 32])], 256, 3, 996)
    x = gu.bf16_tensor(layers[0]["x"])
    dev = [gu.device_paths(lay) for lay in layers]
    ys = [torch.full((3, n + 24), 5.0, dtype=torch.bfloat16, device="cuda") for n in (96, 64)]
    views = [ys[0][:, :96], ys[1][:, :64]]
    lb.linear_forward_siblings(x, [(p[0], p[1] if len(p) > 1 else None) for p in dev], ys=views)
    torch.cuda.synchronize()
    assert bool((ys[0][:, 96:] == 5.0).all()) and bool((ys[1][:, 64:] == 5.0).all())
    for lay, v in zip(layers, views):
        gu.assert_close(gu.bf16_to_f64(v.contiguous()), gu.oracle_y(lay), "strided")
