"""Pins for the fp64 oracle's backward pass (CPU only).

The layer's forward pass (sesamedisk.com, "Samsung LittleBit 13B Model",
"What the method actually computes", Proposition 1) is
    y = sum_p h_p (.) (S_U,p (l_p (.) (S_V,p^T (g_p (.) x)))),
and quantization-aware training runs back through it (littlebitllm.com,
"Pipeline").  ``oracle.backward`` gives the gradients of L = sum dy (.) y with
respect to x and to every path's h, g and l.  Each check below compares it with
something that does not come from the backward code:

* central finite differences of the (separately pinned) forward oracle: y is
  linear in x and in each scale vector on its own, so a central difference is
  exact up to rounding, for every scalar of a tiny layer;
* dx = dy W with the dense W of ``oracle.dense_weight``;
* Euler's identity for functions homogeneous of degree one: sum_o h_o dh_o =
  sum dy (.) y_p for each path's own output y_p, and the same for g and l;
* a Sylvester-Hadamard closed form;
* bitwise invariance under a joint sign flip of a latent pair (u_k, v_k).

The last test plants plausible mistakes and checks that some pin catches each.
"""
import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import random_layer, sylvester


def loss(x, dy, paths):
    return float(np.sum(dy * oracle.forward(x, paths)))


def fd_grads(x, dy, paths, eps=0.5):
    """Central differences of L over every scalar of x, h, g, l."""
    def central(set_value):
        set_value(+eps)
        up = loss(x, dy, paths)
        set_value(-eps)
        dn = loss(x, dy, paths)
        set_value(0.0)
        return (up - dn) / (2 * eps)

    out = {"dx": np.zeros_like(x), "dh": [], "dg": [], "dl": []}
    for m in range(x.shape[0]):
        for i in range(x.shape[1]):
            base = x[m, i]

            def s(d, m=m, i=i, base=base):
                x[m, i] = base + d
            out["dx"][m, i] = central(s)
    for p in paths:
        for name in ("h", "g", "l"):
            vec = p[name]
            grad = np.zeros(len(vec))
            for j in range(len(vec)):
                base = vec[j]

                def s(d, vec=vec, j=j, base=base):
                    vec[j] = base + d
                grad[j] = central(s)
            out["d" + name].append(grad)
    return out


def close(a, b, rtol=1e-10):
    a, b = np.asarray(a, float), np.asarray(b, float)
    return a.shape == b.shape and np.all(np.abs(a - b) <= rtol * max(1.0, np.abs(b).max()))


def _pins_pass(bwd) -> bool:
    """The pins of this file against a (possibly mutated) backward function;
    True only if every one holds."""
    try:
        # finite differences, two paths of different rank, square so that a
        # swapped U and V still has matching shapes
        x, paths = random_layer(np.random.default_rng(3), 6, 6, [3, 2], 3)
        dy = np.random.default_rng(4).standard_normal((3, 6))
        fd = fd_grads(x.copy(), dy, [dict(p) for p in paths])
        b = bwd(x, dy, paths)
        if not close(b["dx"], fd["dx"]):
            return False
        for key in ("dh", "dg", "dl"):
            if len(b[key]) != len(paths) or not all(close(u, v) for u, v in zip(b[key], fd[key])):
                return False
        # dense form and Euler's identity on a wider layer
        x, paths = random_layer(np.random.default_rng(5), 24, 20, [5, 8], 4)
        dy = np.random.default_rng(6).standard_normal((4, 20))
        b = bwd(x, dy, paths)
        if not close(b["dx"], dy @ oracle.dense_weight(paths), 1e-12):
            return False
        for j, p in enumerate(paths):
            lp = float(np.sum(dy * oracle.forward(x, [p])))
            for key, name in (("dh", "h"), ("dg", "g"), ("dl", "l")):
                if not close(np.dot(p[name], b[key][j]), lp, 1e-12):
                    return False
    except (ValueError, IndexError, TypeError):
        return False          # a shape error is a caught mistake too
    return True


def test_backward_matches_finite_differences_and_dense_form():
    assert _pins_pass(oracle.backward)


def test_hadamard_closed_form():
    """S_U = S_V = H_n (rank n), l = c: W = c n diag(h (.) g), so with in = out = n
    dx = c n h g dy, dh_o = c n g_o sum_m dy_mo x_mo, dg_i = c n h_i sum_m x_mi dy_mi."""
    n, c = 32, 0.75
    H = sylvester(n)
    rng = np.random.default_rng(7)
    h, g = np.exp(rng.normal(-1, .5, n)), np.exp(rng.normal(-1, .5, n))
    x, dy = rng.standard_normal((3, n)), rng.standard_normal((3, n))
    b = oracle.backward(x, dy, [dict(su=H, sv=H, h=h, g=g, l=np.full(n, c))])
    assert np.allclose(b["dx"], c * n * h * g * dy, rtol=1e-12, atol=0)
    assert np.allclose(b["dh"][0], c * n * g * np.sum(dy * x, axis=0), rtol=1e-12, atol=1e-14)
    assert np.allclose(b["dg"][0], c * n * h * np.sum(x * dy, axis=0), rtol=1e-12, atol=1e-14)


def test_sign_flip_pair_is_bitwise_invariant():
    """Negating column k of both S_U and S_V leaves every gradient unchanged bit
    for bit (negation is exact and the negated terms meet in a product)."""
    x, paths = random_layer(np.random.default_rng(8), 40, 24, [6, 9], 3)
    dy = np.random.default_rng(9).standard_normal((3, 24))
    b0 = oracle.backward(x, dy, paths)
    flipped = []
    for p in paths:
        su, sv = np.array(p["su"]), np.array(p["sv"])
        su[:, ::2] *= -1
        sv[:, ::2] *= -1
        flipped.append(dict(p, su=su, sv=sv))
    b1 = oracle.backward(x, dy, flipped)
    assert np.array_equal(b0["dx"], b1["dx"])
    for key in ("dh", "dg", "dl"):
        assert all(np.array_equal(u, v) for u, v in zip(b0[key], b1[key]))


def test_zero_tokens_give_zero_scale_gradients():
    _, paths = random_layer(np.random.default_rng(10), 8, 8, [2], 1)
    b = oracle.backward(np.zeros((0, 8)), np.zeros((0, 8)), paths)
    assert b["dx"].shape == (0, 8)
    assert all(np.all(v == 0) for key in ("dh", "dg", "dl") for v in b[key])


def _swap(d, a, b):
    d = dict(d)
    d[a], d[b] = d[b], d[a]
    return d


MUTANTS = {
    "drop_residual_path": lambda x, dy, P: oracle.backward(x, dy, P[:1]),
    "negated_dy": lambda x, dy, P: oracle.backward(x, -dy, P),
    "reversed_output_index": lambda x, dy, P: oracle.backward(x, np.ascontiguousarray(dy[:, ::-1]), P),
    "swap_U_and_V": lambda x, dy, P: oracle.backward(x, dy, [dict(p, su=p["sv"], sv=p["su"]) for p in P]),
    "dh_and_dg_swapped": lambda x, dy, P: _swap(oracle.backward(x, dy, P), "dh", "dg"),
    "dx_without_g": lambda x, dy, P: dict(oracle.backward(x, dy, P), dx=oracle.backward(
        x, dy, [dict(p, g=np.ones(len(p["g"]))) for p in P])["dx"]),
    "paths_swapped_in_dl": lambda x, dy, P: dict(oracle.backward(x, dy, P),
                                                 dl=oracle.backward(x, dy, P)["dl"][::-1]),
    "latent_scale_dropped": lambda x, dy, P: oracle.backward(x, dy, [dict(p, l=np.ones(len(p["l"]))) for p in P]),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name):
    assert not _pins_pass(MUTANTS[name]), f"mutant {name} slipped through the pins"
