"""Benchmark of the LittleBit factored layer's forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {lb,reference}]
                    [--config NAME] [--tokens M] [--no-extras]

Default workload: the Llama-2-7B q_proj shape (4096 -> 4096, eff_bit 1.0,
residual on: two paths of rank 1024) at batch 1.  One step is one pass over
a rotation of distinct copies of the layer's weights (1024 copies, 2.2 GB:
a chain of 1024 layers of this shape), every copy one ``lb_linear_forward``
call (both contractions, both paths), chained on one stream from one CUDA
graph.  The copies span far more than twice the L2 cache and the warm-up
passes over all of them, so every timed call streams its sign bits from HBM.

Printed on rank 0, one JSON line:
  value       whole-job algorithmic HBM GB/s (prefill workloads: TFLOP/s),
              device-timed with CUDA events, max over ranks; us_per_call is
              the timed region over the calls in it
  e2e         the same metric through the C ABI with host buffers
              (lb_linear_forward_host: pinned x in, y out, every call)
  roofline    achieved GB/s of the forward call against the measured HBM peak
  cpu_baseline the fp64 oracle on this host's cores (bounded sample)
  clocks      SM clocks and throttle reasons sampled during the timed region
  prefill     Qwen3-14B gate/up and k/v at 8192 tokens: TFLOP/s, the dominant
              kernel's roofline against the measured bf16 peak, clocks
  backward    Qwen3-14B gate/up at 8192 tokens: lb_linear_backward (dx, dh,
              dg, dl) TFLOP/s against the measured bf16 peak
  decode_block_fused  a Llama-2-7B decoder block's seven linears at 1 token as
              four sibling calls, chained
  dense_baseline      Llama-2-70B gate/up at 1 token against one cuBLAS bf16
              GEMM on the same layer as a dense matrix
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


def source_hash(files=None):
    """Hash of the code of the kernel sources a figure depends on (every
    source when `files` is None): a traffic figure taken on other code is
    stale (comments and layout do not count)."""
    names = sorted(files) if files else sorted(f for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh", ".h")))
    h = hashlib.sha256()
    for f in names:
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
    current code of the sources it names (`sources`: the call's path from the
    ABI to its kernels; all kernel sources when absent): per launch of the
    dominant kernel where the roofline is that kernel's (prefill), else per
    call (decode, whose roofline is the whole call)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{config}/M{tokens}")
    if not e or e.get("source_hash") != source_hash(e.get("sources")):
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
    the region itself ran with its SM clock held down (median below 95 % of
    the maximum); a region whose median clock is at the maximum takes the
    burst figure even if a power-cap reason showed up in some sample."""
    mhz, top = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    capped = mhz is not None and bool(top) and mhz < 0.95 * top
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


def rotation_size(set_bytes, min_sets=1, cap_bytes=4 << 30, max_sets=4096):
    """Weight copies to rotate over: enough that the copies span more than
    twice the L2 cache (every call then finds its weights evicted: between two
    uses of a copy, more than the cache's capacity of other copies is read),
    at least `min_sets`, at most `max_sets` and `cap_bytes` of weights."""
    n = max(-(-2 * L2_BYTES // max(1, set_bytes)) + 1, min_sets)
    return max(1, min(n, max_sets, max(1, cap_bytes // max(1, set_bytes))))


def dense_weight_torch(layer, device):
    """The layer as one dense fp32 matrix W [n_out, n_in] built with plain
    PyTorch ops: W = sum_p diag(h_p) S_U,p diag(l_p) S_V,p^T diag(g_p)
    (sesamedisk.com, "Samsung LittleBit 13B Model", "How low-rank binarization
    works": h scales rows, g columns, l the latent dimension).  The comparison
    arm of the dense baseline; tests check it against the oracle's dense W."""
    import torch
    W = None
    for p in layer["paths"]:
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        su, sv = t(p["su"]).float(), t(p["sv"]).float()
        h, g, l = (t(np.asarray(p[k], dtype=np.float16).view(np.int16)).view(torch.float16).float()
                   for k in ("h", "g", "l"))
        term = (h[:, None] * su * l[None, :]) @ (sv * g[:, None]).t()
        W = term if W is None else W + term
    return W


def time_graph(graph, reps, stream, local, world, device):
    """Replays `graph` `reps` times between CUDA events on `stream`, with a
    barrier and a synchronise on both sides, sampling clocks meanwhile.
    Returns (max-over-ranks ms, clock summary)."""
    import torch
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    with clk:
        start.record(stream)
        for _ in range(reps):
            graph.replay()
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(start.elapsed_time(stop), world, device), clk.summary()


class DeviceLayer:
    """One synthetic workload on the device: its packed paths (and copies of
    them to rotate over), x, y and the workspace."""

    def __init__(self, layer, device, tokens):
        import torch
        import binarized_rank_linear_b200 as lb
        self.lb = lb
        self.layer, self.device, self.tokens = layer, device, tokens
        self.base = []
        for p in layer["paths"]:
            dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
            self.base.append(lb.PackedPath.from_factors(dev(p["su"]), dev(p["sv"]), dev(p["h"]), dev(p["g"]),
                                                        dev(p["l"])))
        self.n_in, self.n_out = layer["n_in"], layer["n_out"]
        self.ranks = [p.rank for p in self.base]
        self.set_bytes = sum(p.u_bits.numel() * 4 + p.vt_bits.numel() * 4 for p in self.base)
        self.nbytes = algorithmic_bytes(self.n_in, self.n_out, self.ranks, tokens)
        self.nflops = algorithmic_flops(self.n_in, self.n_out, self.ranks, tokens)
        self.x = torch.from_numpy(layer["x"].view(np.int16)).to(device).view(torch.bfloat16)
        self.y = torch.empty((tokens, self.n_out), dtype=torch.bfloat16, device=device)
        self.ws = torch.empty(max(16, lb.forward_workspace_bytes(tokens, self.n_in, self.n_out, self.ranks[0],
                                                                 self.ranks[1] if len(self.ranks) > 1 else 0)),
                              dtype=torch.uint8, device=device)
        self.sets = [self.base]

    def rotate(self, nsets):
        lb = self.lb
        clone = lambda p: lb.PackedPath(p.u_bits.clone(), p.vt_bits.clone(), p.h.clone(), p.g.clone(),
                                        p.l.clone(), p.rank)
        self.sets = [self.base] + [[clone(p) for p in self.base] for _ in range(nsets - 1)]

    def call(self, i, x=None, stream=None):
        s = self.sets[i % len(self.sets)]
        self.lb.linear_forward(self.x if x is None else x, s[0], s[1] if len(s) > 1 else None, y=self.y,
                               workspace=self.ws, stream=stream)

    def parity(self, rows):
        """Sampled rows of the last call's y against the fp64 oracle."""
        import torch
        import oracle
        L = self.layer
        ref = oracle.forward(oracle.bf16_bits_to_f64(L["x"][rows]),
                             [dict(su=p["su"], sv=p["sv"], h=oracle.f16_to_f64(p["h"]), g=oracle.f16_to_f64(p["g"]),
                                   l=oracle.f16_to_f64(p["l"])) for p in L["paths"]])
        got = oracle.bf16_bits_to_f64(self.y[torch.from_numpy(rows).to(self.device)].view(torch.int16).cpu()
                                      .numpy().view(np.uint16))
        out = {"rows": int(len(rows)), "rel_l2": float(np.linalg.norm(got - ref) / np.linalg.norm(ref)),
               "max_err_over_max_y": float(np.abs(got - ref).max() / np.abs(ref).max())}
        assert out["rel_l2"] <= 5e-3 and out["max_err_over_max_y"] <= 1e-2, out
        return out


def capture(fn, n, device):
    """A CUDA graph of fn(0), ..., fn(n - 1)."""
    import torch
    cap = torch.cuda.Stream(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        for i in range(n):
            fn(i)
    return g


def time_contractions(d, xs, stream, device, n):
    """Each contraction of the prefill path on its own: lb_latent_forward and
    lb_expand_forward run the same two kernels as lb_linear_forward at these
    token counts.  CUDA graphs of n calls each, over the rotating inputs,
    timed with events on `stream`; flops per contraction from the workload
    table (2 M R n_in and 2 M R n_out)."""
    import torch
    import binarized_rank_linear_b200 as lb
    tokens = d.tokens
    R = sum(d.ranks)
    z = torch.empty((tokens, R), dtype=torch.float16, device=device)
    y = torch.empty((tokens, d.n_out), dtype=torch.bfloat16, device=device)
    two = lambda s: (s[0], s[1] if len(s) > 1 else None)
    lat = lambda i: lb.latent_forward(xs[i % len(xs)], *two(d.sets[i % len(d.sets)]), z=z)
    exp = lambda i: lb.expand_forward(z, *two(d.sets[i % len(d.sets)]), y=y)
    out = {}
    flops = {"contraction_1": 2 * tokens * R * d.n_in, "contraction_2": 2 * tokens * R * d.n_out}
    names = {"contraction_1": "sign_gemm_kernel<1, H, P> (contraction 1, tcgen05)",
             "contraction_2": "sign_gemm_kernel<2, H, P> (contraction 2, tcgen05)"}
    lat(0)
    torch.cuda.synchronize()
    for key, fn in (("contraction_1", lat), ("contraction_2", exp)):
        g = capture(fn, n, device)
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


def measure_prefill(name, args, world, local, device, peaks, tokens=None):
    """One prefill workload (Qwen3-14B linears at 8192 tokens by default):
    the call chained from a CUDA graph, inputs larger than L2 (x rotated over
    copies where x and y together are not), at least `--prefill-seconds` of
    timed calls with the clocks sampled meanwhile; the dominant kernel's
    roofline from its share of the call."""
    import torch
    c = synth.CONFIGS[name]
    tokens = tokens or c.tokens[0]
    d = DeviceLayer(synth.make_config(name, tokens), device, tokens)
    io = 2 * tokens * (d.n_in + d.n_out)
    nx = max(1, min(4, -(-2 * L2_BYTES // io) + 1)) if io <= 2 * L2_BYTES else 1
    xs = [d.x] + [d.x.clone() for _ in range(nx - 1)]
    d.call(0)
    torch.cuda.synchronize()
    assert d.lb.device_status() == d.lb.LB_OK
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([[0, 127, 128, 255, 256, 511, tokens - 1], rng.choice(tokens, 9, replace=False)]))
    parity = d.parity(rows) if not args.no_parity else None
    g = capture(lambda i: d.call(i, x=xs[i % nx]), nx, device)
    for _ in range(max(3, args.warmup)):
        g.replay()
    torch.cuda.synchronize()
    # size the region from one timed replay
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream(device)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    reps = max(3, int(args.prefill_seconds / max(1e-6, e0.elapsed_time(e1) / 1e3)))
    ms, clocks = time_graph(g, reps, stream, local, world, device)
    assert d.lb.device_status() == d.lb.LB_OK
    calls = reps * nx
    per_call_s = ms / 1e3 / calls
    per_kernel = time_contractions(d, xs, stream, device, max(3, min(50, calls)))
    dom = max(per_kernel.values(), key=lambda k: k["share"])
    pk, pk_source = tensor_peak(peaks, clocks)
    achieved = dom["flop"] / (per_call_s * dom["share"]) / 1e12
    return {"workload": workload_name(c, tokens), "tokens": tokens, "calls": calls,
            "l2": "inputs larger than L2" + (" (x rotated over %d copies)" % nx if nx > 1 else ""),
            "us_per_call": per_call_s * 1e6, "value": aggregate(d.nflops / 1e12 * calls, ms / 1e3, world),
            "unit": "TFLOP/s", "algorithmic_flops_per_call": d.nflops,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk, "unit": "TFLOP/s",
                         "frac": achieved / pk, "traffic": load_traffic(name, tokens), "kernel": dom["kernel"],
                         "share_of_call": dom["share"], "call_TFLOP/s": d.nflops / per_call_s / 1e12,
                         "peak_source": pk_source},
            "per_kernel": per_kernel, "parity": parity, "clocks": clocks, "gpu_launches": 2 * calls}


def measure_backward(name, args, world, local, device, peaks, tokens=None):
    """The layer's backward pass (lb_linear_backward: dx and every path's dh,
    dg, dl) on one workload at `tokens` tokens: four tensor-core contractions,
    2 M sum_p r_p (n_in + n_out) flops each pair, so twice the forward pass's
    algorithmic flops.  Chained from a CUDA graph, inputs larger than L2 (x
    and dy rotated over copies where they are not), at least
    `--prefill-seconds` of timed calls with the clocks sampled."""
    import torch
    import binarized_rank_linear_b200 as lb
    c = synth.CONFIGS[name]
    tokens = tokens or c.tokens[-1]
    d = DeviceLayer(synth.make_config(name, tokens), device, tokens)
    rng = np.random.default_rng(7)
    dy = torch.from_numpy(synth.f32_to_bf16_bits(rng.standard_normal((tokens, d.n_out), dtype=np.float32))
                          .view(np.int16)).to(device).view(torch.bfloat16)
    io = 2 * tokens * (d.n_in + d.n_out)
    nx = max(1, min(4, -(-2 * L2_BYTES // io) + 1)) if io <= 2 * L2_BYTES else 1
    xs = [(d.x, dy)] + [(d.x.clone(), dy.clone()) for _ in range(nx - 1)]
    two = lambda s: (s[0], s[1] if len(s) > 1 else None)
    ws = torch.empty(max(16, lb.backward_workspace_bytes(tokens, d.n_in, d.n_out, d.ranks[0],
                                                         d.ranks[1] if len(d.ranks) > 1 else 0)),
                     dtype=torch.uint8, device=device)
    dx = torch.empty((tokens, d.n_in), dtype=torch.bfloat16, device=device)
    call = lambda i: lb.linear_backward(xs[i % nx][0], xs[i % nx][1], *two(d.base), dx=dx, workspace=ws)
    call(0)
    torch.cuda.synchronize()
    assert lb.device_status() == lb.LB_OK
    g = capture(call, nx, device)
    for _ in range(max(3, args.warmup)):
        g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    reps = max(3, int(args.prefill_seconds / max(1e-6, e0.elapsed_time(e1) / 1e3)))
    ms, clocks = time_graph(g, reps, stream, local, world, device)
    assert lb.device_status() == lb.LB_OK
    calls = reps * nx
    per_call_s = ms / 1e3 / calls
    flops = 2 * d.nflops
    pk, pk_source = tensor_peak(peaks, clocks)
    achieved = flops / per_call_s / 1e12
    return {"workload": workload_name(c, tokens) + ", backward (dx, dh, dg, dl)", "tokens": tokens, "calls": calls,
            "us_per_call": per_call_s * 1e6, "algorithmic_flops_per_call": flops,
            "value": aggregate(flops / 1e12 * calls, ms / 1e3, world), "unit": "TFLOP/s",
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk, "unit": "TFLOP/s",
                         "frac": achieved / pk, "traffic": None, "kernel": "whole lb_linear_backward call "
                         "(transpose_bits_kernel (both factors of every path), sign_gemm_kernel<3> x2, "
                         "wgrad_kernel x2 (dh, dg), bf16 sign_gemm_kernel<2> (dx), reduce_partials_kernel)",
                         "peak_source": pk_source},
            "clocks": clocks, "gpu_launches": 7 * calls}


def dense_baseline(d, device, seconds, stream, local, world):
    """The layer as the dense bf16 matrix of dense_weight_torch, applied with
    one cuBLAS GEMM per call (torch.matmul): the comparison behind the pages'
    kernel speedup figure (sesamedisk.com, "Samsung LittleBit 13B Model", "The
    speedup number": a single-kernel speedup over FP16 for one Llama2-70B MLP
    layer).  Copies of W rotate past twice the L2 cache, as the packed weights
    do; calls are chained from a CUDA graph."""
    import torch
    W = dense_weight_torch(d.layer, device).to(torch.bfloat16)
    w_bytes = W.numel() * 2
    nsets = rotation_size(w_bytes, max_sets=64)
    Ws = [W] + [W.clone() for _ in range(nsets - 1)]
    y = torch.empty((d.tokens, W.shape[0]), dtype=torch.bfloat16, device=device)
    n = max(nsets, 32)
    torch.matmul(d.x, Ws[0].t(), out=y)  # warm the cuBLAS handle before capture
    torch.cuda.synchronize()
    g = capture(lambda i: torch.matmul(d.x, Ws[i % nsets].t(), out=y), n, device)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    reps = max(3, int(seconds / max(1e-6, e0.elapsed_time(e1) / 1e3)))
    ms, clocks = time_graph(g, reps, stream, local, world, device)
    del Ws, W
    return {"us_per_call": ms * 1e3 / (reps * n), "kind": "cuBLAS bf16 GEMM (torch.matmul) on the dense weight, "
            "CUDA graphs", "dense_weight_bytes": w_bytes, "weight_sets": nsets, "clocks": clocks}


def time_chained(d, nsets, steps, warmup, device, local, world):
    """Calls chained on one stream from one CUDA graph per pass over `nsets`
    rotating weight copies: `warmup` untimed passes, then `steps` timed
    passes.  Returns (max-over-ranks ms of the timed passes, clocks)."""
    import torch
    d.rotate(nsets)
    g = capture(d.call, nsets, device)
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    ms, clocks = time_graph(g, steps, torch.cuda.current_stream(device), local, world, device)
    del g
    return ms, clocks


def dense_comparison(name, args, world, local, device):
    """The dense baseline beside the LittleBit call on one workload, both
    chained over weights rotated past L2 (Llama-2-70B gate/up at 1 token by
    default: the pages' own kernel comparison)."""
    import torch
    c = synth.CONFIGS[name]
    d = DeviceLayer(synth.make_config(name, c.tokens[0]), device, c.tokens[0])
    nsets = rotation_size(d.set_bytes, min_sets=256)
    ms, _ = time_chained(d, nsets, max(3, args.steps), 3, device, local, world)
    lb_us = ms * 1e3 / (max(3, args.steps) * nsets)
    dense = dense_baseline(d, device, 0.2, torch.cuda.current_stream(device), local, world)
    dense.update(workload=workload_name(c, c.tokens[0]), littlebit_us_per_call=lb_us,
                 speedup=dense["us_per_call"] / lb_us)
    d.sets = [d.base]
    return dense


# A decoder block's linears in the order a forward pass runs them, grouped by
# the input they read (workload names from binarized_rank_linear_b200/synth.py):
# q k v, o, gate up, down.
BLOCKS = {
    "llama2_7b": [["llama2_7b_q"] * 3, ["llama2_7b_q"], ["llama2_7b_gate"] * 2, ["llama2_7b_down"]],
    "qwen3_14b": [["qwen3_14b_qo", "qwen3_14b_kv", "qwen3_14b_kv"], ["qwen3_14b_qo"], ["qwen3_14b_gate"] * 2,
                  ["qwen3_14b_down"]],
}


def measure_block(block, tokens, fused, steps, warmup, world, local, device, seconds=0.0):
    """A whole decoder block's linears at `tokens` tokens, called back to back
    on one stream (each call's launches PDL-chained to the previous one) from
    CUDA graphs; weights rotate past twice the L2 cache.  With `fused` the
    linears that read the same input (q k v; gate up) run as one
    lb_linear_forward_siblings call.  One step is one pass over the block
    copies of a graph; at least `steps` of them are timed (more if needed to
    fill `seconds`)."""
    import torch
    import binarized_rank_linear_b200 as lb

    groups = BLOCKS[block]
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
    nsets = rotation_size(set_bytes, max_sets=64)

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

    def run(i):
        s = sets[i % nsets]
        if not fused:
            for (paths0, x, y, ws), paths in zip(layers, s):
                lb.linear_forward(x, paths[0], paths[1] if len(paths) > 1 else None, y=y, workspace=ws)
            return
        for gi, (a, b) in enumerate(zip(gstart[:-1], gstart[1:])):
            lb.linear_forward_siblings(gx[gi], [(s[k][0], s[k][1] if len(s[k]) > 1 else None) for k in range(a, b)],
                                       ys=[layers[k][2] for k in range(a, b)], workspace=gws[gi])

    run(0)
    torch.cuda.synchronize()
    assert lb.device_status() == lb.LB_OK
    per_graph = max(1, min(2 * nsets, 64))
    g = capture(run, per_graph, device)
    for _ in range(max(1, warmup)):
        g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(device)
    reps = max(1, steps)
    if seconds > 0:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        reps = max(reps, int(seconds / max(1e-6, e0.elapsed_time(e1) / 1e3)))
    ms, clocks = time_graph(g, reps, stream, local, world, device)
    assert lb.device_status() == lb.LB_OK
    blocks = reps * per_graph
    per_block_s = ms / 1e3 / blocks
    decode = tokens <= DECODE_MAX_TOKENS
    peaks = load_peaks()
    achieved = (nbytes / per_block_s / 1e9) if decode else (nflops / per_block_s / 1e12)
    pk, pk_source = (peaks["hbm"], peaks["source"]) if decode else tensor_peak(peaks, clocks)
    launches_per_block = 2 * (len(groups) if fused and tokens <= 128 else len(seq))
    return {"workload": "%s block (%s) at %d tokens" % (block, ", ".join(seq), tokens), "tokens": tokens,
            "linears": len(seq), "weight_sets": nsets, "blocks": blocks, "ms": ms,
            "calls": ("one lb_linear_forward_siblings call per input group (%d)" % len(groups))
            if fused else "one lb_linear_forward call per linear",
            "launch": "CUDA graphs of %d blocks" % per_graph,
            "us_per_block": per_block_s * 1e6, "algorithmic_bytes_per_block": nbytes,
            "algorithmic_flops_per_block": nflops,
            "value": aggregate(((nbytes / 1e9) if decode else (nflops / 1e12)) * blocks, ms / 1e3, world),
            "unit": "GB/s" if decode else "TFLOP/s",
            "roofline": {"bound": "hbm" if decode else "tensor", "achieved": achieved, "peak": pk,
                         "unit": "GB/s" if decode else "TFLOP/s", "frac": achieved / pk, "traffic": None,
                         "peak_source": pk_source},
            "clocks": clocks, "gpu_launches": launches_per_block * blocks}


def run_block(args, world, rank, local):
    """--block: one step is one pass of a whole decoder block's linears."""
    import torch
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    tokens = args.tokens or 1
    r = measure_block(args.block, tokens, args.fused, args.steps, args.warmup, world, local, device)
    if rank != 0:
        return
    out = {"metric": "decoder block of LittleBit linears: us/block, " + r["unit"], "value": r["value"],
           "unit": r["unit"], "n_gpus": world, "steps": r["blocks"], "warmup": args.warmup,
           "ms_per_step": r["ms"] / r["blocks"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "bf16", "data": "synthetic",
           "config": {k: r[k] for k in ("workload", "tokens", "linears", "weight_sets", "calls", "launch")},
           "us_per_block": r["us_per_block"], "algorithmic_bytes_per_block": r["algorithmic_bytes_per_block"],
           "algorithmic_flops_per_block": r["algorithmic_flops_per_block"], "roofline": r["roofline"],
           "clocks": r["clocks"], "gpu_launches": r["gpu_launches"], "impl": "lb"}
    print(json.dumps(out), flush=True)


NUMERICS = ("bf16 x and y, fp16 scales, fp32 accumulation (1-4 tokens: fp32 throughout; more tokens: tensor-core "
            "operands bf16 in contraction 1, fp16 in contraction 2)")


def run_lb(args, world, rank, local):
    import torch
    import binarized_rank_linear_b200 as lb

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    c = synth.CONFIGS[args.config]
    tokens = args.tokens or c.tokens[0]
    decode = tokens <= DECODE_MAX_TOKENS
    peaks = load_peaks()
    d = DeviceLayer(synth.make_config(args.config, tokens), device, tokens)
    nbytes, nflops = d.nbytes, d.nflops
    stream = torch.cuda.current_stream(device)

    # parity of the benchmarked configuration against the oracle (sampled rows)
    d.call(0)
    torch.cuda.synchronize()
    assert lb.device_status() == lb.LB_OK
    parity = None
    if rank == 0 and not args.no_parity:
        parity = d.parity(np.arange(tokens) if tokens <= 8 else np.linspace(0, tokens - 1, 8).astype(int))

    # One step is one pass over `nsets` distinct copies of the layer's weights
    # (a chain of nsets layers of this shape), chained on one stream from one
    # CUDA graph.  The copies span more than twice the L2 cache, and the
    # warm-up passes over all of them, so no call of the timed region finds
    # its weights in L2.
    io_bytes = 2 * tokens * (d.n_in + d.n_out)
    nsets = 1 if io_bytes > 2 * L2_BYTES else rotation_size(d.set_bytes, min_sets=args.min_sets)
    ms_max, clocks = time_chained(d, nsets, args.steps, args.warmup, device, local, world)
    calls = args.steps * nsets
    per_call_s = ms_max / 1e3 / calls
    units = nbytes / 1e9 if decode else nflops / 1e12
    value = aggregate(units * calls, ms_max / 1e3, world)
    assert lb.device_status() == lb.LB_OK

    # isolated calls: cold L2 before each
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device)
    iso = []
    for i in range(20):
        flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        d.call(i)
        e1.record(stream)
        torch.cuda.synchronize()
        iso.append(e0.elapsed_time(e1) * 1e3)
    iso_us = statistics.median(iso)
    del flush

    # end to end through the C ABI with host buffers (lb_linear_forward_host):
    # the same steps (passes over the weight copies), every call bringing its
    # x in from pinned host memory and its y back to pinned host memory
    # inside the one call.  Two ways to issue them: the calls captured once
    # into a CUDA graph per step (as a serving loop issues its decode steps;
    # each replay moves every call's x and y across the host link again), and
    # eagerly from Python, one ctypes call at a time
    x_host = torch.empty_like(d.x, device="cpu").pin_memory()
    x_host.copy_(d.x.cpu())
    y_host = torch.empty((tokens, d.n_out), dtype=torch.bfloat16).pin_memory()

    def call_host(i):
        s = d.sets[i % nsets]
        lb.linear_forward_host(x_host, s[0], s[1] if len(s) > 1 else None, y_host, d.x, d.y, d.ws)

    for i in range(nsets):
        call_host(i)
    torch.cuda.synchronize()
    hg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(hg, stream=torch.cuda.Stream(device), capture_error_mode="relaxed"):
        for i in range(nsets):
            call_host(i)
    for _ in range(args.warmup):
        hg.replay()
    torch.cuda.synchronize()
    y_host.fill_(0)
    e2e_ms, _ = time_graph(hg, args.steps, stream, local, world, device)
    e2e_ok = bool(torch.equal(y_host.to(device), d.y)) if tokens <= 128 else None  # the last call's y arrived
    del hg
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(calls):
        call_host(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    eager_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    e2e_value = aggregate(units * calls, e2e_ms / 1e3, world)
    d.sets = [d.base]
    torch.cuda.empty_cache()

    # the default run also measures prefill (the metric's TFLOP/s half), a
    # whole decoder block of fused sibling calls at batch 1, and the dense
    # baseline of the pages' kernel comparison
    prefill = block = dense = backward = None
    extras = set() if args.no_extras else set(args.extras.split(","))
    if "prefill" in extras:
        prefill = {}
        for name in args.prefill.split(",") if args.prefill else []:
            prefill[name] = measure_prefill(name, args, world, local, device, peaks)
            torch.cuda.empty_cache()
    if "backward" in extras:
        backward = {}
        for name in args.backward.split(",") if args.backward else []:
            backward[name] = measure_backward(name, args, world, local, device, peaks)
            torch.cuda.empty_cache()
    if "block" in extras:
        block = measure_block("llama2_7b", 1, True, args.steps, args.warmup, world, local, device, seconds=0.1)
        torch.cuda.empty_cache()
    if "dense" in extras:
        dense = dense_comparison("llama2_70b_gate", args, world, local, device)
        torch.cuda.empty_cache()
    if args.dense_baseline and dense is None:
        dense = dense_comparison(args.config, args, world, local, device)

    if rank != 0:
        return
    if decode or tokens <= 128:
        achieved = nbytes / per_call_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm"], "unit": "GB/s",
                "frac": achieved / peaks["hbm"], "traffic": load_traffic(args.config, tokens),
                "kernel": kernel_label(tokens, c.rank * c.paths * (c.n_in + c.n_out)),
                "peak_source": peaks["source"]}
    else:
        pk, pk_source = tensor_peak(peaks, clocks)
        per_kernel = time_contractions(d, [d.x], stream, device, max(3, min(args.steps, 50)))
        dom = max(per_kernel.values(), key=lambda k: k["share"])
        achieved = dom["flop"] / (per_call_s * dom["share"]) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk, "unit": "TFLOP/s", "frac": achieved / pk,
                "traffic": load_traffic(args.config, tokens), "kernel": dom["kernel"],
                "share_of_call": dom["share"], "call_TFLOP/s": nflops / per_call_s / 1e12, "peak_source": pk_source}
    cpu = None
    if world == 1 and not args.no_cpu:
        import oracle
        per, nb, nf, desc = oracle_sample(synth.make_config(args.config, min(tokens, 64)), args.cpu_seconds)
        cpu = {"value": (nb / per / 1e9) if decode else (nf / per / 1e12), "unit": "GB/s" if decode else "TFLOP/s",
               "cores": oracle.num_threads(), "kind": "oracle", "sample": desc}
    set_mb = nsets * d.set_bytes / 1e6
    out = {"metric": METRIC, "value": value, "unit": "GB/s" if decode else "TFLOP/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
           "numerics": NUMERICS, "data": "synthetic",
           "config": {"workload": workload_name(c, tokens), "tokens": tokens, "weight_sets": nsets,
                      "step": "one pass over %d distinct weight copies: %d lb_linear_forward calls chained on one "
                              "stream from one CUDA graph" % (nsets, nsets),
                      "l2": ("weights rotated over %.0f MB > 2x L2; warm-up passes over every copy" % set_mb)
                      if set_mb * 1e6 > 2 * L2_BYTES else
                      ("inputs larger than L2" if io_bytes > 2 * L2_BYTES else "weights within L2 (%.0f MB)" % set_mb),
                      "parallelism": "replicas" if world > 1 else "single GPU"},
           "us_per_call": per_call_s * 1e6, "calls_timed": calls, "us_per_call_isolated_cold_l2": iso_us,
           "algorithmic_bytes_per_call": nbytes, "algorithmic_flops_per_call": nflops,
           "roofline": roof, "cpu_baseline": cpu, "parity": parity, "clocks": clocks,
           "e2e": {"value": e2e_value, "unit": "GB/s" if decode else "TFLOP/s",
                   "h2d_bytes_per_step": 2 * tokens * d.n_in * nsets, "d2h_bytes_per_step": 2 * tokens * d.n_out * nsets,
                   "us_per_call": e2e_ms * 1e3 / calls, "calls": calls,
                   "call": "lb_linear_forward_host (pinned host x and y; " + (
                       "x gathered by a kernel in one pass, y written in place by the last kernel)" if tokens <= 128 else
                       "copied through device buffers inside the call)") +
                   ", %d calls per step captured in a CUDA graph" % nsets,
                   "y_host_matches_device_call": e2e_ok,
                   "eager": {"value": aggregate(units * calls, eager_ms / 1e3, world),
                             "us_per_call": eager_ms * 1e3 / calls,
                             "call": "the same calls issued one at a time from Python"}},
           "gpu_launches": 2 * calls,  # contraction 1 + contraction 2 per call, decode and prefill
           "impl": "lb"}
    if prefill:
        out["prefill"] = prefill
    if backward:
        out["backward"] = backward
    if block is not None:
        out["decode_block_fused"] = block
    if dense is not None:
        out["dense_baseline"] = dense
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["lb", "reference"], default="lb")
    ap.add_argument("--config", default="llama2_7b_q", choices=sorted(synth.CONFIGS))
    ap.add_argument("--tokens", type=int, default=0, help="default: the config's first token count")
    ap.add_argument("--min-sets", type=int, default=1024,
                    help="decode: weight copies per step at least (more if needed to pass 2x L2)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--prefill", default="qwen3_14b_gate,qwen3_14b_kv",
                    help="prefill workloads measured beside the main line (comma-separated)")
    ap.add_argument("--prefill-seconds", type=float, default=0.3)
    ap.add_argument("--backward", default="qwen3_14b_gate",
                    help="workloads whose backward pass is measured beside the main line (comma-separated)")
    ap.add_argument("--extras", default="prefill,backward,block,dense",
                    help="measurements beside the main line: any of prefill, backward, block, dense")
    ap.add_argument("--no-extras", action="store_true", help="none of the --extras")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-parity", action="store_true")
    ap.add_argument("--block", choices=sorted(BLOCKS), default=None,
                    help="time a whole decoder block's linears chained (tokens default 1)")
    ap.add_argument("--fused", action="store_true",
                    help="with --block: linears that share their input run as one siblings call")
    ap.add_argument("--dense-baseline", action="store_true",
                    help="with --no-extras: also time a cuBLAS bf16 GEMM on this workload's dense weight")
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
