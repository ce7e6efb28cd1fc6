"""Host-side logic of bench.py: the algorithmic byte and FLOP counts of the
workload table, and the replica aggregation (max over ranks) on two gloo
processes."""
import os

import pytest

import bench
from binarized_rank_linear_b200 import synth

# per-call algorithmic bytes / flops of the workload table (packed sign bits +
# fp16 scales + bf16 x and y; flops of the two contractions)
EXPECTED = {
    ("tiny", 1): (4160, 32768),
    ("llama2_7b_q", 1): (2150400, 33554432),
    ("llama2_7b_q", 8): (2265088, 268435456),
    ("llama2_7b_gate", 1): (3114624, 48332800),
    ("llama2_7b_gate", 32): (4051072, 48332800 * 32),
    ("llama2_70b_gate", 1): (2876544, 42467328),
    ("qwen3_14b_gate", 8192): (375320832, 803158884352),
}


@pytest.mark.parametrize("key", sorted(EXPECTED))
def test_algorithmic_counts(key):
    name, m = key
    c = synth.CONFIGS[name]
    ranks = [c.rank] * c.paths
    nb, nf = EXPECTED[key]
    assert bench.algorithmic_bytes(c.n_in, c.n_out, ranks, m) == nb
    assert bench.algorithmic_flops(c.n_in, c.n_out, ranks, m) == nf


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 30.0][rank]
        mx = bench.max_over_ranks(ms, world)
        bench.barrier(world)
        q.put((rank, mx, bench.aggregate(100.0, mx / 1e3, world)))
    finally:
        dist.destroy_process_group()


def test_replicas_take_the_slowest_rank():
    import socket

    import torch.multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, value in res:
        assert mx == 30.0                       # max over ranks
        assert value == pytest.approx(2 * 100.0 / 0.030)   # both ranks' units / slowest time


def test_reference_arm_non_zero_ranks_exit(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--steps", "3", "--warmup", "3"])
    assert capsys.readouterr().out == ""


def test_blocks_are_the_models_linears():
    """--block: every entry names a workload of the table, and the linears'
    shapes chain as a decoder block does (attention in -> model width, MLP
    up -> intermediate width, down -> model width)."""
    for name, groups in bench.BLOCKS.items():
        linears = [synth.CONFIGS[w] for grp in groups for w in grp]
        for grp in groups:                                        # a group shares its input
            assert len({synth.CONFIGS[w].n_in for w in grp}) == 1 and len(grp) <= 4
        assert len(linears) == 7
        width = linears[0].n_in
        assert all(c.n_in == width for c in linears[:3])           # q, k, v read the block input
        assert linears[3].n_out == width                          # o writes the model width
        gate, up, down = linears[4:]
        assert gate.n_in == up.n_in == width and gate.n_out == up.n_out == down.n_in
        assert down.n_out == width


def test_kernel_labels_follow_the_dispatch():
    q7 = 2 * 1024 * (4096 + 4096)      # Llama-2-7B q_proj sign bits
    gate7 = 2 * 800 * (4096 + 11008)   # Llama-2-7B gate/up
    assert "small1_kernel" in bench.kernel_label(1, gate7) and "small1_kernel" in bench.kernel_label(2, gate7)
    assert "small1_kernel" in bench.kernel_label(4, q7) and "small1_kernel" in bench.kernel_label(3, gate7)
    assert "mid_gemm_kernel" in bench.kernel_label(4, gate7)
    assert "mid_gemm_kernel" in bench.kernel_label(5) and "mid_gemm_kernel" in bench.kernel_label(128)
    assert "sign_gemm_kernel" in bench.kernel_label(129)


def test_tensor_peak_follows_the_sampled_clocks():
    """The sustained (power-capped) cuBLAS figure is the denominator only when
    the timed region itself ran with its clock held down; otherwise the burst
    figure is, even if a power-cap reason appeared in some sample."""
    peaks = dict(hbm=6542.4, bf16=1651.4, bf16_sustained=1401.9, source="measured")
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": [], "samples": 12}
    assert bench.tensor_peak(peaks, at_max) == (1651.4, "measured (burst)")
    capped_at_max = dict(at_max, reasons=["sw_power_cap"])
    assert bench.tensor_peak(peaks, capped_at_max) == (1651.4, "measured (burst)")
    slow = dict(at_max, sm_mhz=1492.0, reasons=["sw_power_cap"])
    assert bench.tensor_peak(peaks, slow) == (1401.9, "measured (sustained)")
    assert bench.tensor_peak(peaks, {"error": "nvml unavailable"}) == (1651.4, "measured (burst)")


def test_source_hash_sees_code_not_comments():
    """Traffic figures stay valid across comment edits and go stale on any
    change to the code itself."""
    a = "int f(int x) { return x + 1; }  // one\n/* two */\n"
    b = "// one, reworded\nint f(int x)\n{\n    return x + 1; /* three */\n}\n"
    c = "int f(int x) { return x + 2; }\n"
    assert bench.source_code(a) == bench.source_code(b)
    assert bench.source_code(a) != bench.source_code(c)
    assert "one" not in bench.source_code(a) and "two" not in bench.source_code(a)


def test_source_hash_covers_the_named_sources():
    """A figure's hash covers the sources it names (all of them when none are
    named), in a fixed order."""
    names = sorted(f for f in os.listdir(bench.CSRC) if f.endswith((".cu", ".cuh", ".h")))
    assert bench.source_hash() == bench.source_hash(names)
    sub = ["lb_gemv.cu", "lb_common.cuh"]
    assert bench.source_hash(sub) == bench.source_hash(list(reversed(sub)))
    assert bench.source_hash(sub) != bench.source_hash(names)


@pytest.mark.parametrize("n_in,n_out,ranks", [(256, 512, [64, 32]), (96, 64, [32])])
def test_dense_baseline_weight_is_the_oracles(n_in, n_out, ranks):
    """The dense comparison arm multiplies by W built with PyTorch ops
    (dense_weight_torch); it must be the oracle's dense W of the same layer
    (fp32 build: within fp32 rounding of the fp64 product), and its bf16 copy,
    which the GEMM reads, within bf16 rounding."""
    import numpy as np
    import oracle
    import torch
    layer = synth.make_layer(n_in, n_out, ranks, 1, config_id=1300 + n_in)
    P = [dict(su=p["su"], sv=p["sv"], h=oracle.f16_to_f64(p["h"]), g=oracle.f16_to_f64(p["g"]),
              l=oracle.f16_to_f64(p["l"])) for p in layer["paths"]]
    ref = oracle.dense_weight(P)
    W = bench.dense_weight_torch(layer, "cpu")
    assert tuple(W.shape) == (n_out, n_in) and W.dtype == torch.float32
    got = W.double().numpy()
    scale = np.abs(ref).max()
    assert np.abs(got - ref).max() <= 1e-5 * scale
    wb = W.to(torch.bfloat16).double().numpy()
    assert np.all(np.abs(wb - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6 * scale)


def test_rotation_spans_twice_l2():
    for set_bytes in (4160, 2150400, 6_100_000, 400_000_000):
        n = bench.rotation_size(set_bytes, min_sets=1)
        if n * set_bytes <= (4 << 30) and n < 4096:
            assert n * set_bytes > 2 * bench.L2_BYTES
    assert bench.rotation_size(2150400, min_sets=1024) == 1024
    assert bench.rotation_size(10 ** 9, min_sets=1024) == 4   # capped by 4 GB of weights
