"""Benchmark of the LittleBit factored layer's forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {lb,reference}]
                    [--config NAME] [--tokens M]

One step is one ``lb_linear_forward`` call (both contractions, both paths)
over one batch of synthetic input.  Default workload: the Llama-2-7B q_proj
shape (4096 -> 4096, eff_bit 1.0, residual on: two paths of rank 1024) at
batch 1.  Steps rotate over enough copies of the weights that the set is
larger than twice the L2 cache, so every call streams its sign bits from HBM;
the calls run back to back from CUDA graphs (the chained, per-layer number).

Printed on rank 0, one JSON line:
  value       whole-job algorithmic HBM GB/s (prefill workloads: TFLOP/s),
              device-timed with CUDA events, max over ranks
  e2e         the same metric through the C ABI with host buffers
              (lb_linear_forward_host: pinned x copied in, y copied out,
              every step)
  roofline    achieved GB/s of the forward call against the measured HBM peak
  cpu_baseline the fp64 oracle on this host's cores (bounded sample)
  clocks      SM clocks and throttle reasons sampled during the timed region
With ``--impl reference`` the fp64 CPU oracle is timed instead (rank 0 only).
Multi-GPU runs are independent replicas (the layer needs no exchange at this
scale): every rank runs the same workload on its own GPU.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from binarized_rank_linear_b200 import synth  # noqa: E402

METRIC = "LittleBitLinear µs/call & HBM GB/s (batch 1); prefill TFLOP/s; % of roofline"
DECODE_MAX_TOKENS = 32
L2_BYTES = 126 * 1024 * 1024
CSRC = os.path.join(ROOT, "binarized_rank_linear_b200", "csrc")


# ---------------------------------------------------------------- workload arithmetic

def algorithmic_bytes(n_in, n_out, ranks, tokens):
    """Packed sign bits + fp16 scales + bf16 x and y, per call."""
    bits = sum(r * (n_in + n_out) for r in ranks) // 8
    scales = sum(2 * (n_in + n_out + r) for r in ranks)
    return bits + scales + 2 * tokens * n_in + 2 * tokens * n_out


def algorithmic_flops(n_in, n_out, ranks, tokens):
    """The two sign contractions: 2 * M * sum_p r_p (n_in + n_out)."""
    return 2 * tokens * sum(r * (n_in + n_out) for r in ranks)


def workload_name(c, tokens):
    return (f"{c.name}: {c.n_in}->{c.n_out}, eff_bit {c.eff_num}/{c.eff_den}, "
            f"{c.paths} path(s) x rank {c.rank}, {tokens} token(s)")


def source_code(text):
    """A C/CUDA source with its comments removed and whitespace collapsed: what
    the compiler sees (the kernel sources hold no "//" or "/*" in a string)."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def source_hash():
    """Hash of every kernel source's code: a traffic figure taken on other code
    is stale (comments and layout do not count)."""
    h = hashlib.sha256()
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(CSRC, f)) as fh:
                h.update(f.encode() + b"\0" + source_code(fh.read()).encode())
    return h.hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sustained=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def load_traffic(config, tokens):
    """DRAM bytes from a committed ncu summary, only if it was taken on the
    current kernel sources: per launch of the dominant kernel where the
    roofline is that kernel's (prefill), else per call (decode, whose
    roofline is the whole call)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{config}/M{tokens}")
    if not e or e.get("source_hash") != source_hash():
        return None
    return e.get("dram_bytes_per_launch", e.get("dram_bytes_per_call"))


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML in a thread."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index, interval=0.001):
        self.samples, self.reasons, self.ok = [], 0, False
        self.interval = interval
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + uuid if not uuid.startswith("GPU-") else uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that instead of clocks
            self.err = str(e)
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.interval)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        r = [name for bit, name in self.REASONS.items() if self.reasons & bit and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": r, "samples": len(self.samples)}


def tensor_peak(peaks, clocks):
    """The tensor-core denominator for a timed region: the sustained figure is
    cuBLAS bf16 with the clock settled under the power cap, so it applies when
    the region ran power-capped too (the cap reported, or the median SM clock
    well below its maximum); otherwise the burst figure applies."""
    reasons = clocks.get("reasons") or []
    mhz, top = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    capped = "sw_power_cap" in reasons or (mhz is not None and top and mhz < 0.9 * top)
    return (peaks["bf16_sustained"], peaks["source"] + " (sustained)") if capped else \
        (peaks["bf16"], peaks["source"] + " (burst)")


# ---------------------------------------------------------------- distributed plumbing

def dist_setup(gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value, world, device="cpu"):
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(per_rank_units, seconds_max, world):
    """Whole-job throughput: every rank processes the same units; the job takes
    the slowest rank's time."""
    return per_rank_units * world / seconds_max


# ---------------------------------------------------------------- CPU oracle timing

def oracle_sample(layer, budget_s, min_runs=2):
    """Time the oracle on a bounded sample of the workload: a contiguous block
    of latent indices k of every path (the layer is a sum over k, so this is an
    exact sub-problem), sized so one run takes about budget_s / min_runs.
    Returns (seconds per run, algorithmic bytes per run, flops per run,
    description)."""
    import oracle
    x = oracle.bf16_bits_to_f64(layer["x"])
    full = [dict(su=p["su"], sv=p["sv"], h=oracle.f16_to_f64(p["h"]), g=oracle.f16_to_f64(p["g"]),
                 l=oracle.f16_to_f64(p["l"])) for p in layer["paths"]]
    n_in, n_out, M = layer["n_in"], layer["n_out"], x.shape[0]
    rank = full[0]["su"].shape[1]

    def sliced(kb):
        return [dict(p, su=np.ascontiguousarray(p["su"][:, :kb]), sv=np.ascontiguousarray(p["sv"][:, :kb]),
                     l=p["l"][:kb]) for p in full]

    kb = min(rank, 32)
    t0 = time.perf_counter()
    oracle.forward(x, sliced(kb))
    t1 = time.perf_counter() - t0
    target = budget_s / min_runs
    kb = int(max(1, min(rank, kb * target / max(t1, 1e-6))))
    paths = sliced(kb)
    runs, t_total = 0, 0.0
    while runs < min_runs or t_total < budget_s * 0.5:
        t0 = time.perf_counter()
        oracle.forward(x, paths)
        t_total += time.perf_counter() - t0
        runs += 1
        if t_total > budget_s * 2:
            break
    per = t_total / runs
    nb = algorithmic_bytes(n_in, n_out, [kb] * len(paths), M)
    nf = algorithmic_flops(n_in, n_out, [kb] * len(paths), M)
    desc = (f"{M} token(s), latent indices 0..{kb - 1} of {rank} in each of {len(paths)} path(s) "
            f"({runs} run(s), {t_total:.1f} s)")
    return per, nb, nf, desc


def run_reference(args, world, rank):
    """--impl reference: the fp64 CPU oracle on the host cores, rank 0 only."""
    if rank != 0:
        return
    import oracle
    c = synth.CONFIGS[args.config]
    tokens = args.tokens or c.tokens[0]
    decode = tokens <= DECODE_MAX_TOKENS
    layer = synth.make_config(args.config, min(tokens, 64))
    budget = 150.0 / max(1, args.steps + args.warmup)
    per, nb, nf, desc = oracle_sample(layer, max(budget, 0.05), min_runs=1)
    for _ in range(args.warmup):
        pass  # the sample run above is the warm-up
    t_steps = per * args.steps
    value = (nb / per / 1e9) if decode else (nf / per / 1e12)
    unit = "GB/s" if decode else "TFLOP/s"
    if tokens > 64:
        desc += f" (first 64 of {tokens} tokens)"
    out = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": per * 1e3, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": workload_name(c, tokens), "tokens": tokens},
           "impl": "reference",
           "cpu_baseline": {"value": value, "unit": unit, "cores": oracle.num_threads(), "kind": "oracle",
                            "sample": desc},
           "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
           "timed_seconds": t_steps}
    print(json.dumps(out), flush=True)


# ---------------------------------------------------------------- the GPU arm

def kernel_label(tokens, sign_bits=0):
    """The kernels a call runs, as the library dispatches: 1-4 tokens on CUDA
    cores unless 3-4 tokens x sign bits (sum of r (in + out)) pass 80 M."""
    if tokens <= 2 or (tokens <= 4 and tokens * sign_bits <= 80_000_000):
        return "lb_linear_forward call: small1_kernel + small2_kernel (CUDA cores, PDL-chained)"
    if tokens <= 128:
        return ("lb_linear_forward call: mid_gemm_kernel<1> + mid_gemm_kernel<2> "
                "(tcgen05, sign matrix as the 128-row operand, PDL-chained)")
    return "lb_linear_forward call: sign_gemm_kernel<1> + sign_gemm_kernel<2> (tcgen05, persistent)"


def dense_baseline(layer, x, steps, stream, device):
    """The layer as the dense bf16 matrix W = sum_p diag(h_p) S_U diag(l_p)
    S_V^T diag(g_p), applied with one cuBLAS GEMM per call (torch.matmul): the comparison the pages' kernel speedup
    figure makes (littlebitllm.com, "How small"; the single-kernel speedup
    quoted for a Llama2-70B layer).  W is built with plain PyTorch ops on the
    GPU; copies rotate past twice the L2 cache, as the packed weights do."""
    import torch
    W = None
    for p in layer["paths"]:
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        su, sv = t(p["su"]).float(), t(p["sv"]).float()
        h, g, l = (t(p[k].view(np.int16)).view(torch.float16).float() for k in ("h", "g", "l"))
        term = (h[:, None] * su * l[None, :]) @ (sv * g[:, None]).t()
        W = term if W is None else W + term
    W = W.to(torch.bfloat16)
    w_bytes = W.numel() * 2
    nsets = max(1, min(64, -(-2 * L2_BYTES // w_bytes) + 1))
    Ws = [W] + [W.clone() for _ in range(nsets - 1)]
    y = torch.empty((x.shape[0], W.shape[0]), dtype=torch.bfloat16, device=device)
    per_graph = max(nsets, 32)
    cap = torch.cuda.Stream(device)
    torch.matmul(x, Ws[0].t(), out=y)  # warm the cuBLAS handle before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        for i in range(per_graph):
            torch.matmul(x, Ws[i % nsets].t(), out=y)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    reps = max(1, min(200, steps // per_graph))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (reps * per_graph)
    return {"us_per_call": us, "kind": "cuBLAS bf16 GEMM (torch.matmul) on the dense weight, CUDA graphs",
            "dense_weight_bytes": w_bytes, "weight_sets": nsets}


# A decoder block's linears in the order a forward pass runs them, grouped by
# the input they read (workload names from binarized_rank_linear_b200/synth.py):
# q k v, o, gate up, down.
BLOCKS = {
    "llama2_7b": [["llama2_7b_q"] * 3, ["llama2_7b_q"], ["llama2_7b_gate"] * 2, ["llama2_7b_down"]],
    "qwen3_14b": [["qwen3_14b_qo", "qwen3_14b_kv", "qwen3_14b_kv"], ["qwen3_14b_qo"], ["qwen3_14b_gate"] * 2,
                  ["qwen3_14b_down"]],
}


def run_block(args, world, rank, local):
    """One step is a whole decoder block's linears at `tokens` tokens, called
    back to back on one stream (each call's launches PDL-chained to the
    previous one) from CUDA graphs; weights rotate past twice the L2 cache.
    With --fused the linears that read the same input (q k v; gate up) run
    as one lb_linear_forward_siblings call."""
    import torch
    import binarized_rank_linear_b200 as lb

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    tokens = args.tokens or 1
    groups = BLOCKS[args.block]
    seq = [name for grp in groups for name in grp]
    layers, nbytes, nflops = [], 0, 0
    for j, name in enumerate(seq):
        c = synth.CONFIGS[name]
        ranks = [c.rank] * c.paths
        nbytes += algorithmic_bytes(c.n_in, c.n_out, ranks, tokens)
        nflops += algorithmic_flops(c.n_in, c.n_out, ranks, tokens)
        lay = synth.make_config(name, tokens, seed=j)
        paths = []
        for p in lay["paths"]:
            dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
            paths.append(lb.PackedPath.from_factors(dev(p["su"]), dev(p["sv"]), dev(p["h"]), dev(p["g"]), dev(p["l"])))
        x = torch.from_numpy(lay["x"].view(np.int16)).to(device).view(torch.bfloat16)
        y = torch.empty((tokens, c.n_out), dtype=torch.bfloat16, device=device)
        ws = torch.empty(max(16, lb.forward_workspace_bytes(tokens, c.n_in, c.n_out, c.rank,
                                                            c.rank if c.paths > 1 else 0)),
                         dtype=torch.uint8, device=device)
        layers.append((paths, x, y, ws))
    set_bytes = sum(p.u_bits.numel() * 4 + p.vt_bits.numel() * 4 for lay in layers for p in lay[0])
    nsets = max(1, min(64, -(-2 * L2_BYTES // set_bytes) + 1))

    def clone(p):
        return lb.PackedPath(p.u_bits.clone(), p.vt_bits.clone(), p.h.clone(), p.g.clone(), p.l.clone(), p.rank)

    sets = [[lay[0] for lay in layers]] + [[[clone(p) for p in lay[0]] for lay in layers] for _ in range(nsets - 1)]

    # fused: one shared x and workspace per group
    gstart = np.cumsum([0] + [len(grp) for grp in groups])
    gx, gws = [], []
    for a, b in zip(gstart[:-1], gstart[1:]):
        gx.append(layers[a][1])
        spec = [(layers[k][0][0], layers[k][0][1] if len(layers[k][0]) > 1 else None) for k in range(a, b)]
        gws.append(torch.empty(max(16, lb.siblings_workspace_bytes(tokens, gx[-1].shape[1], spec)),
                               dtype=torch.uint8, device=device))

    def block(i):
        s = sets[i % nsets]
        if not args.fused:
            for (paths0, x, y, ws), paths in zip(layers, s):
                lb.linear_forward(x, paths[0], paths[1] if len(paths) > 1 else None, y=y, workspace=ws)
            return
        for gi, (a, b) in enumerate(zip(gstart[:-1], gstart[1:])):
            lb.linear_forward_siblings(gx[gi], [(s[k][0], s[k][1] if len(s[k]) > 1 else None) for k in range(a, b)],
                                       ys=[layers[k][2] for k in range(a, b)], workspace=gws[gi])

    block(0)
    torch.cuda.synchronize()
    assert lb.device_status() == lb.LB_OK
    per_graph = max(1, min(2 * nsets, 64))
    cap = torch.cuda.Stream(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        for i in range(per_graph):
            block(i)
    for _ in range(max(1, args.warmup // per_graph)):
        g.replay()
    torch.cuda.synchronize()
    reps = max(1, args.steps // per_graph)
    stream = torch.cuda.current_stream(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    with clk:
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    steps = reps * per_graph
    per_block_s = ms / 1e3 / steps
    assert lb.device_status() == lb.LB_OK
    if rank != 0:
        return
    decode = tokens <= DECODE_MAX_TOKENS
    peaks = load_peaks()
    achieved = (nbytes / per_block_s / 1e9) if decode else (nflops / per_block_s / 1e12)
    pk, pk_source = (peaks["hbm"], peaks["source"]) if decode else tensor_peak(peaks, clk.summary())
    out = {"metric": "decoder block of LittleBit linears: us/block, " + ("HBM GB/s" if decode else "TFLOP/s"),
           "value": aggregate(((nbytes / 1e9) if decode else (nflops / 1e12)) * steps, ms / 1e3, world),
           "unit": "GB/s" if decode else "TFLOP/s", "n_gpus": world, "steps": steps, "warmup": args.warmup,
           "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "f16", "data": "synthetic",
           "config": {"workload": "%s block (%s) at %d tokens" % (args.block, ", ".join(seq), tokens),
                      "tokens": tokens, "linears": len(seq), "weight_sets": nsets,
                      "calls": ("one lb_linear_forward_siblings call per input group (%d)" % len(groups))
                      if args.fused else "one lb_linear_forward call per linear",
                      "launch": "CUDA graphs of %d blocks" % per_graph},
           "us_per_block": per_block_s * 1e6, "algorithmic_bytes_per_block": nbytes,
           "algorithmic_flops_per_block": nflops,
           "roofline": {"bound": "hbm" if decode else "tensor", "achieved": achieved, "peak": pk,
                        "unit": "GB/s" if decode else "TFLOP/s", "frac": achieved / pk, "traffic": None,
                        "peak_source": pk_source},
           "clocks": clk.summary(),
           "gpu_launches": 2 * (len(groups) if args.fused and tokens <= 4 else len(seq)) * steps, "impl": "lb"}
    print(json.dumps(out), flush=True)


def time_contractions(sets, x, tokens, c, stream, device, n):
    """Each contraction of the prefill path on its own: lb_latent_forward and
    lb_expand_forward run the same two kernels as lb_linear_forward at these
    token counts.  CUDA graphs of n calls each, over the rotating weights,
    timed with events on `stream`; flops per contraction from the workload
    table (2 M R n_in and 2 M R n_out)."""
    import torch
    import binarized_rank_linear_b200 as lb
    R = sum(p.rank for p in sets[0])
    z = torch.empty((tokens, R), dtype=torch.float16, device=device)
    y = torch.empty((tokens, c.n_out), dtype=torch.bfloat16, device=device)
    two = lambda s: (s[0], s[1] if len(s) > 1 else None)
    lat = lambda i: lb.latent_forward(x, *two(sets[i % len(sets)]), z=z)
    exp = lambda i: lb.expand_forward(z, *two(sets[i % len(sets)]), y=y)
    out = {}
    cap = torch.cuda.Stream(device)
    flops = {"contraction_1": 2 * tokens * R * c.n_in, "contraction_2": 2 * tokens * R * c.n_out}
    names = {"contraction_1": "sign_gemm_kernel<1, H, P> (contraction 1, tcgen05)",
             "contraction_2": "sign_gemm_kernel<2, H, P> (contraction 2, tcgen05)"}
    lat(0)
    torch.cuda.synchronize()
    for key, fn in (("contraction_1", lat), ("contraction_2", exp)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            for i in range(n):
                fn(i)
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / n
        out[key] = {"kernel": names[key], "flop": flops[key], "us_alone": us, "TFLOP/s_alone": flops[key] / us / 1e6}
        del g
    total = sum(v["us_alone"] for v in out.values())
    for v in out.values():
        v["share"] = v["us_alone"] / total
    return out


def run_lb(args, world, rank, local):
    import torch
    import binarized_rank_linear_b200 as lb

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    c = synth.CONFIGS[args.config]
    tokens = args.tokens or c.tokens[0]
    ranks = [c.rank] * c.paths
    decode = tokens <= DECODE_MAX_TOKENS
    nbytes = algorithmic_bytes(c.n_in, c.n_out, ranks, tokens)
    nflops = algorithmic_flops(c.n_in, c.n_out, ranks, tokens)
    layer = synth.make_config(args.config, tokens)

    # weights: one packed set through the C ABI, then copies so the rotation
    # covers more than twice the L2 cache
    base = []
    for p in layer["paths"]:
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        base.append(lb.PackedPath.from_factors(dev(p["su"]), dev(p["sv"]), dev(p["h"]), dev(p["g"]), dev(p["l"])))
    set_bytes = sum(p.u_bits.numel() * 4 + p.vt_bits.numel() * 4 for p in base)
    io_bytes = 2 * tokens * (c.n_in + c.n_out)
    nsets = 1 if io_bytes > 2 * L2_BYTES else max(1, min(512, -(-2 * L2_BYTES // set_bytes) + 1))

    def clone(p):
        return lb.PackedPath(p.u_bits.clone(), p.vt_bits.clone(), p.h.clone(), p.g.clone(), p.l.clone(), p.rank)

    sets = [base] + [[clone(p) for p in base] for _ in range(nsets - 1)]
    x = torch.from_numpy(layer["x"].view(np.int16)).to(device).view(torch.bfloat16)
    y = torch.empty((tokens, c.n_out), dtype=torch.bfloat16, device=device)
    ws = torch.empty(max(16, lb.forward_workspace_bytes(tokens, c.n_in, c.n_out, c.rank,
                                                        c.rank if c.paths > 1 else 0)),
                     dtype=torch.uint8, device=device)

    def call(i, stream=None):
        s = sets[i % nsets]
        lb.linear_forward(x, s[0], s[1] if len(s) > 1 else None, y=y, workspace=ws, stream=stream)

    # parity of the benchmarked configuration against the oracle (sampled rows)
    call(0)
    torch.cuda.synchronize()
    assert lb.device_status() == lb.LB_OK
    parity = None
    if rank == 0 and not args.no_parity:
        import oracle
        rows = np.arange(tokens) if tokens <= 8 else np.linspace(0, tokens - 1, 8).astype(int)
        ref = oracle.forward(oracle.bf16_bits_to_f64(layer["x"][rows]),
                             [dict(su=p["su"], sv=p["sv"], h=oracle.f16_to_f64(p["h"]),
                                   g=oracle.f16_to_f64(p["g"]), l=oracle.f16_to_f64(p["l"]))
                              for p in layer["paths"]])
        got = oracle.bf16_bits_to_f64(y[torch.from_numpy(rows).to(device)].view(torch.int16).cpu().numpy()
                                      .view(np.uint16))
        parity = {"rows": int(len(rows)),
                  "rel_l2": float(np.linalg.norm(got - ref) / np.linalg.norm(ref)),
                  "max_err_over_max_y": float(np.abs(got - ref).max() / np.abs(ref).max())}
        assert parity["rel_l2"] <= 5e-3 and parity["max_err_over_max_y"] <= 1e-2, parity

    # CUDA graphs of consecutive calls over the rotating weight sets
    per_graph = max(1, min(nsets * (2 if nsets < 64 else 1), 512)) if decode else 1
    cap_stream = torch.cuda.Stream(device)

    def capture(n, start):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap_stream):
            for i in range(n):
                call(start + i)
        return g

    graph = capture(per_graph, 0)
    tail_n = args.steps % per_graph
    tail = capture(tail_n, 0) if tail_n else None
    full_graphs = args.steps // per_graph

    def run_steps(n_full, tail_graph):
        for _ in range(n_full):
            graph.replay()
        if tail_graph is not None:
            tail_graph.replay()

    # warm-up
    wf, wt = divmod(args.warmup, per_graph)
    run_steps(wf, capture(wt, 0) if wt else None)
    torch.cuda.synchronize()

    # timed region
    stream = torch.cuda.current_stream(device)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    with clk:
        start.record(stream)
        run_steps(full_graphs, tail)
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = start.elapsed_time(stop)
    ms_max = max_over_ranks(ms, world, device)
    per_call_s = ms_max / 1e3 / args.steps
    units = nbytes / 1e9 if decode else nflops / 1e12
    value = aggregate(units * args.steps, ms_max / 1e3, world)
    assert lb.device_status() == lb.LB_OK

    # isolated calls: cold L2 before each
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device)
    iso = []
    for i in range(20):
        flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call(i)
        e1.record(stream)
        torch.cuda.synchronize()
        iso.append(e0.elapsed_time(e1) * 1e3)
    iso_us = statistics.median(iso)
    del flush

    # end to end through the C ABI with host buffers (lb_linear_forward_host):
    # every step copies x in from pinned host memory, runs the layer and
    # copies y back to pinned host memory, all inside the one call
    x_host = torch.empty_like(x, device="cpu").pin_memory()
    x_host.copy_(x.cpu())
    y_host = torch.empty((tokens, c.n_out), dtype=torch.bfloat16).pin_memory()
    e2e_steps = min(args.steps, max(50, args.e2e_steps))

    def call_host(i):
        s = sets[i % nsets]
        lb.linear_forward_host(x_host, s[0], s[1] if len(s) > 1 else None, y_host, x, y, ws)

    for i in range(min(20, e2e_steps)):
        call_host(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        call_host(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    e2e_value = aggregate(units * e2e_steps, e2e_ms / 1e3, world)

    dense = dense_baseline(layer, x, args.steps, stream, device) if args.dense_baseline else None
    per_kernel = (time_contractions(sets, x, tokens, c, stream, device, max(3, min(args.steps, 50)))
                  if not decode and tokens > 128 else None)

    if rank != 0:
        return
    peaks = load_peaks()
    if decode:
        achieved = nbytes / per_call_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm"], "unit": "GB/s",
                "frac": achieved / peaks["hbm"], "traffic": load_traffic(args.config, tokens),
                "kernel": kernel_label(tokens, c.rank * c.paths * (c.n_in + c.n_out)),
                "peak_source": peaks["source"]}
    else:
        pk, pk_source = tensor_peak(peaks, clk.summary())
        if per_kernel is not None:
            # the dominant kernel: its share of the call comes from timing each
            # contraction alone (after the timed region, where the clocks under
            # the power cap have settled lower, so only the ratio is used); its
            # duration is that share of the live per-call time
            dom = max(per_kernel.values(), key=lambda k: k["share"])
            achieved = dom["flop"] / (per_call_s * dom["share"]) / 1e12
            roof = {"bound": "tensor", "achieved": achieved, "peak": pk, "unit": "TFLOP/s",
                    "frac": achieved / pk, "traffic": load_traffic(args.config, tokens),
                    "kernel": dom["kernel"], "share_of_call": dom["share"],
                    "call_TFLOP/s": nflops / per_call_s / 1e12,
                    "peak_source": pk_source}
        else:
            achieved = nflops / per_call_s / 1e12
            roof = {"bound": "tensor", "achieved": achieved, "peak": pk, "unit": "TFLOP/s",
                    "frac": achieved / pk, "traffic": load_traffic(args.config, tokens),
                    "kernel": kernel_label(tokens, c.rank * c.paths * (c.n_in + c.n_out)),
                    "peak_source": pk_source}
    cpu = None
    if world == 1 and not args.no_cpu:
        import oracle
        per, nb, nf, desc = oracle_sample(synth.make_config(args.config, min(tokens, 64)), args.cpu_seconds)
        cpu = {"value": (nb / per / 1e9) if decode else (nf / per / 1e12), "unit": "GB/s" if decode else "TFLOP/s",
               "cores": oracle.num_threads(), "kind": "oracle", "sample": desc}
    out = {"metric": METRIC, "value": value, "unit": "GB/s" if decode else "TFLOP/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
           "data": "synthetic",
           "config": {"workload": workload_name(c, tokens), "tokens": tokens, "weight_sets": nsets,
                      "l2": ("weights rotated over %.0f MB > 2x L2" % (nsets * set_bytes / 1e6)) if nsets > 1
                      else "inputs larger than L2",
                      "launch": "CUDA graphs of %d back-to-back calls" % per_graph,
                      "parallelism": "replicas" if world > 1 else "single GPU"},
           "us_per_call": per_call_s * 1e6, "us_per_call_isolated_cold_l2": iso_us,
           "algorithmic_bytes_per_call": nbytes, "algorithmic_flops_per_call": nflops,
           "roofline": roof, "per_kernel": per_kernel, "cpu_baseline": cpu, "parity": parity,
           "clocks": clk.summary(),
           "e2e": {"value": e2e_value, "unit": "GB/s" if decode else "TFLOP/s",
                   "h2d_bytes_per_step": 2 * tokens * c.n_in, "d2h_bytes_per_step": 2 * tokens * c.n_out,
                   "steps": e2e_steps, "call": "lb_linear_forward_host (pinned host x and y; " + (
                       "x gathered by a kernel in one pass, y written in place by the last kernel)" if tokens <= 128 else
                       "copied through device buffers inside the call)")},
           "gpu_launches": 2 * args.steps,  # contraction 1 + contraction 2 per call, decode and prefill
           "impl": "lb"}
    if dense is not None:
        dense["speedup"] = dense["us_per_call"] / (per_call_s * 1e6)
        out["dense_baseline"] = dense
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=2000)
    ap.add_argument("--impl", choices=["lb", "reference"], default="lb")
    ap.add_argument("--config", default="llama2_7b_q", choices=sorted(synth.CONFIGS))
    ap.add_argument("--tokens", type=int, default=0, help="default: the config's first token count")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--e2e-steps", type=int, default=5000)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-parity", action="store_true")
    ap.add_argument("--block", choices=sorted(BLOCKS), default=None,
                    help="time a whole decoder block's linears chained (tokens default 1)")
    ap.add_argument("--fused", action="store_true",
                    help="with --block: linears that share their input run as one siblings call")
    ap.add_argument("--dense-baseline", action="store_true",
                    help="also time a cuBLAS bf16 GEMM on the reconstructed dense weight (same tokens)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores; other ranks exit at once
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        (run_block if args.block else run_lb)(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
