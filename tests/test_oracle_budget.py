"""Pins for the bit-budget rank rule (CPU only).

The budget (sesamedisk.com, "How low-rank binarization works": "the rank sets
the bit budget"; littlebitllm.com, "How small": linear layers only, scale
vectors not counted; with residual compensation the two paths share it,
sesamedisk.com, same section) is  paths * r * (n_in + n_out) <= eff * n_in * n_out.
The rank per path is the largest such r, rounded down to a multiple of the
alignment.  Expected ranks are the workload table's literal values.
"""
from fractions import Fraction

import pytest

import oracle
from binarized_rank_linear_b200 import synth


@pytest.mark.parametrize("name", sorted(synth.CONFIGS))
def test_config_ranks(name):
    c = synth.CONFIGS[name]
    assert oracle.rank_for_budget(c.n_in, c.n_out, c.eff_num, c.eff_den, c.paths, 32) == c.rank


@pytest.mark.parametrize("name", sorted(synth.CONFIGS))
def test_budget_identity(name):
    c = synth.CONFIGS[name]
    eff = Fraction(c.eff_num, c.eff_den)
    budget = eff * c.n_in * c.n_out
    used = c.paths * c.rank * (c.n_in + c.n_out)
    assert used <= budget                                   # never above the budget
    assert c.paths * (c.rank + 32) * (c.n_in + c.n_out) > budget   # the next multiple would be
    assert Fraction(used, c.n_in * c.n_out) <= eff          # achieved bpw <= eff


def test_exact_quotients_need_exact_arithmetic():
    """For Qwen3-14B q/o and gate at 0.55 the quotient is an exact integer (704,
    1088): the budget is met with no slack, so any rounding below the exact
    value would make the floor drop a whole alignment step.  The rule works on
    the fraction eff_num / eff_den to rule that out."""
    assert Fraction(55, 100) * 5120 * 5120 / (2 * (5120 + 5120)) == 704
    assert Fraction(55, 100) * 5120 * 17408 / (2 * (5120 + 17408)) == 1088
    assert oracle.rank_for_budget(5120, 5120, 55, 100, 2, 32) == 704
    assert oracle.rank_for_budget(5120, 17408, 55, 100, 2, 32) == 1088


def test_unaligned_rule():
    assert oracle.rank_for_budget(4096, 11008, 55, 100, 2, 1) == 820
    assert oracle.rank_for_budget(8192, 28672, 1, 10, 2, 1) == 318
    assert oracle.rank_for_budget(5120, 1024, 55, 100, 2, 1) == 234


def test_size_ratio_at_055_bpw():
    """littlebitllm.com hero: 0.55 bits per weight, linear layers ~29x smaller
    than BF16: 16 / 0.55 = 29.09."""
    assert round(16 / 0.55) == 29


# Public Llama-2 dimensions (hidden, intermediate, layers, kv dim, vocab).  They
# are not on the pages; the pages give only the resulting sizes.
LLAMA2 = {"7b": (4096, 11008, 32, 4096), "13b": (5120, 13824, 40, 5120),
          "70b": (8192, 28672, 80, 1024)}
PAGE_GB = {"7b": 0.63, "13b": 0.84, "70b": 1.98}   # sesamedisk.com, "The real result"
PAGE_FP16_GB = {"7b": 13.49, "13b": 26.06, "70b": 138.0}


@pytest.mark.parametrize("model", sorted(LLAMA2))
def test_footprint_at_01_bpw(model):
    """Sizes at 0.1 bpw from the rank rule: sign bits of every linear layer
    (two paths, unaligned rank), fp16 scales (n_in + n_out + r per path),
    embeddings and lm_head in bf16, norms in bf16.  Agrees with the page's
    figures to within 3 %."""
    d, f, L, kv = LLAMA2[model]
    vocab = 32000
    shapes = [(d, d), (d, kv), (d, kv), (d, d), (d, f), (d, f), (f, d)]
    bits = 0
    scale_bytes = 0
    dense = 0
    for n_in, n_out in shapes:
        r = oracle.rank_for_budget(n_in, n_out, 1, 10, 2, 1)
        bits += 2 * r * (n_in + n_out)
        scale_bytes += 2 * 2 * (n_in + n_out + r)
        dense += n_in * n_out
    emb = 2 * vocab * d * 2
    norms = (2 * L + 1) * d * 2
    total = L * (bits / 8 + scale_bytes) + emb + norms
    fp16 = L * dense * 2 + emb + norms
    assert abs(fp16 / 1e9 - PAGE_FP16_GB[model]) / PAGE_FP16_GB[model] < 0.01
    assert abs(total / 1e9 - PAGE_GB[model]) / PAGE_GB[model] < 0.03
