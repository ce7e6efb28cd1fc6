"""Failure handling on the GPU, made to happen without faulting the device.

The fault tests of the library's test plan: every device-side wait in the
kernels is bounded in time, and a wait that runs out must end in a status the
host can read, with the context still usable.  Here a test hook
(lb_debug_inject_stall) shortens the tcgen05 decode kernels' limit to 1 ms and
makes one producer warp of the first CTA skip its arrival on its first stage
barrier.  The MMA thread's wait on that barrier runs out; the kernel winds
down (drains its copies and MMAs, frees its tensor memory) and records
LB_ERR_DEVICE_TIMEOUT.  Nothing traps, nothing hangs: the next call on the
same stream runs normally and matches the oracle.
"""
import numpy as np
import pytest

import binarized_rank_linear_b200 as lb
from binarized_rank_linear_b200 import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("tokens,n_in,n_out,ranks", [(16, 256, 384, [64, 32]), (40, 4096, 4096, [1024, 1024])])
def test_bounded_wait_times_out_and_the_context_survives(tokens, n_in, n_out, ranks):
    import torch
    layer = synth.make_layer(n_in, n_out, ranks, tokens, config_id=1500 + n_in)
    paths = gu.device_paths(layer)
    x = gu.bf16_tensor(layer["x"])
    y = torch.empty((tokens, n_out), dtype=torch.bfloat16, device="cuda")
    assert lb.device_status() == lb.LB_OK
    lb.debug_inject_stall(True, 1_000_000)
    try:
        lb.linear_forward(x, paths[0], paths[1], y=y)     # enqueued with the hook on
    finally:
        lb.debug_inject_stall(False)
    torch.cuda.synchronize()                              # returns: the kernels ended
    assert lb.device_status() == lb.LB_ERR_DEVICE_TIMEOUT
    assert lb.device_status() == lb.LB_OK                 # reading cleared it
    # the same stream, the same buffers: a normal call
    lb.linear_forward(x, paths[0], paths[1], y=y)
    torch.cuda.synchronize()
    assert lb.device_status() == lb.LB_OK
    gu.assert_close(gu.bf16_to_f64(y), gu.oracle_y(layer), f"after the timeout M={tokens}")


def test_hook_rejects_bad_limits():
    with pytest.raises(lb.LbError):
        lb.debug_inject_stall(True, 10)            # below 1 us
    with pytest.raises(lb.LbError):
        lb.debug_inject_stall(True, 5_000_000_000)  # above the default 2 s
    lb.debug_inject_stall(False)
