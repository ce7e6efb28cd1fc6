"""lb_linear_forward_fixed_scratch on the GPU: the decode forward pass with
the library's fixed device scratch instead of a caller workspace.

The file name sorts last, so in a full run these calls come after every other
test has used the library; the tests pass alone too.  Each case makes two
calls in a row and compares both, bit for bit, with lb_linear_forward on the
same inputs (the same kernels run; only the scratch differs), and checks the
result against the fp64 oracle.
"""
import numpy as np
import pytest

import binarized_rank_linear_b200 as lb
from binarized_rank_linear_b200 import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

CASES = [("tiny", 1), ("llama2_7b_q", 1), ("llama2_7b_q", 8), ("llama2_7b_gate", 4), ("llama2_7b_down", 16),
         ("qwen3_14b_gate", 32), ("llama2_70b_down", 1)]


@pytest.mark.parametrize("name,tokens", CASES)
def test_two_calls_match_the_workspace_entry(name, tokens):
    import torch
    layer = synth.make_config(name, tokens)
    paths = gu.device_paths(layer)
    res = paths[1] if len(paths) > 1 else None
    x = gu.bf16_tensor(layer["x"])
    y_ref = lb.linear_forward(x, paths[0], res)
    y1 = lb.linear_forward_fixed_scratch(x, paths[0], res)
    y2 = torch.full_like(y1, float("nan"))
    lb.linear_forward_fixed_scratch(x, paths[0], res, y=y2)
    torch.cuda.synchronize()
    assert lb.device_status() == lb.LB_OK
    ref_bits = gu.bf16_bits(y_ref)
    assert np.array_equal(gu.bf16_bits(y1), ref_bits)
    assert np.array_equal(gu.bf16_bits(y2), ref_bits)
    gu.assert_close(gu.bf16_to_f64(y1), gu.oracle_y(layer), f"{name} M={tokens}")


def test_refused_shapes_write_nothing():
    import torch
    layer = synth.make_config("llama2_7b_q", 33)
    paths = gu.device_paths(layer)
    x = gu.bf16_tensor(layer["x"])
    y = torch.full((33, 4096), 3.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lb.LbError) as e:
        lb.linear_forward_fixed_scratch(x, paths[0], paths[1], y=y)
    assert e.value.status == lb.LB_ERR_UNSUPPORTED_SHAPE
    torch.cuda.synchronize()
    assert bool((y == 3.0).all())


def test_scratch_too_small_writes_nothing():
    """32 tokens (inside the token limit) on two paths of rank 16384: the
    latent needs 2 MiB, more than the fixed array holds, so the call is
    refused on the host with LB_ERR_WORKSPACE_TOO_SMALL and y keeps its
    canary values."""
    import torch
    n, r, tokens = 256, 16384, 32
    assert lb.forward_workspace_bytes(tokens, n, n, r, r) > (1 << 20)
    layer = synth.make_layer(n, n, [r, r], tokens, config_id=1201)
    paths = gu.device_paths(layer)
    x = gu.bf16_tensor(layer["x"])
    y = torch.full((tokens, n), 3.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lb.LbError) as e:
        lb.linear_forward_fixed_scratch(x, paths[0], paths[1], y=y)
    assert e.value.status == lb.LB_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    assert bool((y == 3.0).all())
    assert lb.device_status() == lb.LB_OK
