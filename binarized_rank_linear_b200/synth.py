"""Seeded synthetic inputs for the LittleBit layer workloads.

This module only draws random numbers.  It holds none of the layer's
arithmetic, imports neither the CUDA binding nor the oracle, and is the one
piece of code that both sides of a parity check share: the same arrays go to
the oracle (as int8 signs and widened scales) and to the CUDA library (packed
on the device by ``lb_pack_signs``).

Workloads (shapes from the pages: Llama-2-7B / 70B layers, sesamedisk.com,
"The real result" and "The speedup number"; Qwen3-14B, littlebitllm.com,
"Releases"; the model dimensions themselves are the public configs):

=================  ==========  =========  ======  =====  ======================
name               n_in        n_out      eff     paths  rank per path
=================  ==========  =========  ======  =====  ======================
tiny               256         256        1/4     1      32
llama2_7b_q        4096        4096       1       2      1024
llama2_7b_gate     4096        11008      0.55    2      800
llama2_7b_down     11008       4096       0.55    2      800
llama2_70b_gate    8192        28672      0.1     2      288
llama2_70b_down    28672       8192       0.1     2      288
qwen3_14b_qo       5120        5120       0.55    2      704
qwen3_14b_kv       5120        1024       0.55    2      224
qwen3_14b_gate     5120        17408      0.55    2      1088
qwen3_14b_down     17408       5120       0.55    2      1088
=================  ==========  =========  ======  =====  ======================

The ranks are literal here on purpose: the rank rule is checked against them,
not used to make them.

Value distributions (seed 0 unless a caller says otherwise):

* x ~ N(0, 1), rounded to bf16 (round to nearest even);
* signs iid Bernoulli(0.5) -> int8 +-1;
* scales: ``tiny``: |N(0,1)| * 0.05 + 0.01 -> fp16; all others:
  exp(N(-3, 0.5)) -> fp16 (lognormal), drawn independently per path and
  vector.

Every tensor has its own stream:
``numpy.random.default_rng(SeedSequence([seed, config_id, tensor_id]))`` with
tensor ids x = 0 and, for path p (0-based), sv = 1 + 5p, su = 2 + 5p,
g = 3 + 5p, l = 4 + 5p, h = 5 + 5p.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class LayerConfig:
    name: str
    config_id: int
    n_in: int
    n_out: int
    eff_num: int
    eff_den: int
    paths: int
    rank: int
    tokens: tuple
    scales: str  # "tiny" or "lognormal"


CONFIGS = {c.name: c for c in [
    LayerConfig("tiny", 0, 256, 256, 1, 4, 1, 32, (1,), "tiny"),
    LayerConfig("llama2_7b_q", 1, 4096, 4096, 1, 1, 2, 1024, (1, 8), "lognormal"),
    LayerConfig("llama2_7b_gate", 2, 4096, 11008, 55, 100, 2, 800, (1, 4, 16, 32), "lognormal"),
    LayerConfig("llama2_7b_down", 3, 11008, 4096, 55, 100, 2, 800, (1, 4, 16, 32), "lognormal"),
    LayerConfig("llama2_70b_gate", 4, 8192, 28672, 1, 10, 2, 288, (1,), "lognormal"),
    LayerConfig("llama2_70b_down", 5, 28672, 8192, 1, 10, 2, 288, (1,), "lognormal"),
    LayerConfig("qwen3_14b_qo", 6, 5120, 5120, 55, 100, 2, 704, (8192,), "lognormal"),
    LayerConfig("qwen3_14b_kv", 7, 5120, 1024, 55, 100, 2, 224, (8192,), "lognormal"),
    LayerConfig("qwen3_14b_gate", 8, 5120, 17408, 55, 100, 2, 1088, (8192,), "lognormal"),
    LayerConfig("qwen3_14b_down", 9, 17408, 5120, 55, 100, 2, 1088, (8192,), "lognormal"),
]}


def rng_for(seed: int, config_id: int, tensor_id: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, config_id, tensor_id]))


def f32_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even.  Inputs
    here are finite draws, so NaN handling is not needed."""
    b = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32)
    rounded = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def draw_x(rng: np.random.Generator, tokens: int, n_in: int) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal((tokens, n_in), dtype=np.float32))


def draw_signs(rng: np.random.Generator, rows: int, cols: int) -> np.ndarray:
    b = rng.integers(0, 2, size=(rows, cols), dtype=np.int8)
    return (1 - 2 * b).astype(np.int8)


def draw_scale(rng: np.random.Generator, n: int, kind: str) -> np.ndarray:
    if kind == "tiny":
        v = np.abs(rng.standard_normal(n)) * 0.05 + 0.01
    elif kind == "lognormal":
        v = np.exp(rng.normal(-3.0, 0.5, size=n))
    else:
        raise ValueError(kind)
    return v.astype(np.float16)


def make_layer(n_in: int, n_out: int, ranks, tokens: int, *, seed: int = 0,
               config_id: int = 1000, scales: str = "lognormal") -> dict:
    """Draw one layer and one input batch.

    Returns ``{"x": uint16 bf16 bits [tokens, n_in], "paths": [ {"sv": int8
    [n_in, r], "su": int8 [n_out, r], "g": f16 [n_in], "l": f16 [r], "h": f16
    [n_out]} ... ]}``.
    """
    paths = []
    for p, r in enumerate(ranks):
        base = 1 + 5 * p
        paths.append(dict(
            sv=draw_signs(rng_for(seed, config_id, base + 0), n_in, r),
            su=draw_signs(rng_for(seed, config_id, base + 1), n_out, r),
            g=draw_scale(rng_for(seed, config_id, base + 2), n_in, scales),
            l=draw_scale(rng_for(seed, config_id, base + 3), r, scales),
            h=draw_scale(rng_for(seed, config_id, base + 4), n_out, scales),
        ))
    x = draw_x(rng_for(seed, config_id, 0), tokens, n_in)
    return dict(x=x, paths=paths, n_in=n_in, n_out=n_out)


def make_config(name: str, tokens: int | None = None, *, seed: int = 0) -> dict:
    """Draw the named workload (see the table above) at ``tokens`` tokens
    (default: the config's first token count)."""
    c = CONFIGS[name]
    m = c.tokens[0] if tokens is None else tokens
    return make_layer(c.n_in, c.n_out, [c.rank] * c.paths, m, seed=seed,
                      config_id=c.config_id, scales=c.scales)
