"""Pins for the fp64 oracle's forward pass and dense form (CPU only).

Each check compares the oracle with something that does not come from the
oracle: a hand-worked example, a closed form, a brute-force sum in a different
order, the rank of the product, or an exact invariance.  The last test plants
plausible mistakes into the oracle's inputs (a dropped residual path, swapped
scales, swapped or transposed factors, a missing latent scale) and checks that
some pin catches every one of them.

The layer (sesamedisk.com, "Samsung LittleBit 13B Model", "What the method
actually computes", Proposition 1):
    Y = ((((X (.) g) V_sign) (.) l) U_sign^T) (.) h,
summed over the primary and the residual path ("How low-rank binarization
works", last paragraph).
"""

import numpy as np
import pytest

import oracle
from tests.conftest import load_golden


def sylvester(n: int) -> np.ndarray:
    """Sylvester Hadamard matrix H_n (n a power of two), H H^T = n I."""
    H = np.array([[1]], dtype=np.int8)
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]]).astype(np.int8)
    return H


def hand_paths(fx):
    p1 = dict(sv=fx["p1_sv"], su=fx["p1_su"], g=fx["p1_g"], l=fx["p1_l"], h=fx["p1_h"])
    p2 = dict(sv=fx["p2_sv"], su=fx["p2_su"], g=fx["p2_g"], l=fx["p2_l"], h=fx["p2_h"])
    return p1, p2


def brute_force(x, paths):
    """Literal quadruple sum y[m,o] = sum_p sum_k sum_i h_o su[o,k] l_k sv[i,k]
    g_i x[m,i], in pure Python, k outermost inside each path (a different
    order from the oracle's)."""
    x = np.asarray(x, dtype=np.float64)
    M, n_in = x.shape
    n_out = len(paths[0]["h"])
    y = [[0.0] * n_out for _ in range(M)]
    for m in range(M):
        for o in range(n_out):
            acc = 0.0
            for p in paths:
                su, sv = np.asarray(p["su"]), np.asarray(p["sv"])
                h, g, l = (np.asarray(p[k], dtype=np.float64) for k in ("h", "g", "l"))
                for k in range(su.shape[1]):
                    inner = 0.0
                    for i in range(n_in):
                        inner += float(sv[i, k]) * float(g[i]) * float(x[m, i])
                    acc += float(h[o]) * float(su[o, k]) * float(l[k]) * inner
            y[m][o] = acc
    return np.array(y)


def random_layer(rng, n_in, n_out, ranks, M, unit_scales=False, int_x=False):
    paths = []
    for r in ranks:
        p = dict(sv=(1 - 2 * rng.integers(0, 2, (n_in, r))).astype(np.int8),
                 su=(1 - 2 * rng.integers(0, 2, (n_out, r))).astype(np.int8))
        for name, n in (("g", n_in), ("l", r), ("h", n_out)):
            if unit_scales:
                p[name] = np.ones(n)
            else:
                p[name] = np.exp(rng.normal(-1.0, 0.5, n)).astype(np.float16).astype(np.float64)
        paths.append(p)
    if int_x:
        x = rng.integers(-1, 2, (M, n_in)).astype(np.float64)
    else:
        x = rng.standard_normal((M, n_in)).astype(np.float32).astype(np.float64)
    return x, paths


# ---------------------------------------------------------------- hand example

def test_hand_example_forward():
    fx = load_golden("forward_hand.txt")
    p1, p2 = hand_paths(fx)
    y = oracle.forward(np.array(fx["x"], dtype=np.float64), [p1, p2])
    assert np.array_equal(y, np.array(fx["y"], dtype=np.float64))
    y1 = oracle.forward(np.array(fx["x"], dtype=np.float64), [p1])
    assert np.array_equal(y1, np.array(fx["y_path1"], dtype=np.float64))


def test_hand_example_dense():
    fx = load_golden("forward_hand.txt")
    p1, p2 = hand_paths(fx)
    assert np.array_equal(oracle.dense_weight([p1]), np.array(fx["W_path1"], float))
    assert np.array_equal(oracle.dense_weight([p1, p2]), np.array(fx["W"], float))


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("n", [32, 256])
def test_hadamard_closed_form(n):
    """S_U = S_V = H_n, l = c: W = c n diag(h (.) g), so y = c n h (.) g (.) x."""
    rng = np.random.default_rng(10 + n)
    H = sylvester(n)
    c = 0.375
    h = np.exp(rng.normal(-3, 0.5, n)).astype(np.float16).astype(np.float64)
    g = np.exp(rng.normal(-3, 0.5, n)).astype(np.float16).astype(np.float64)
    x = rng.standard_normal((3, n)).astype(np.float32).astype(np.float64)
    y = oracle.forward(x, [dict(su=H, sv=H, h=h, g=g, l=np.full(n, c))])
    expect = c * n * h[None, :] * g[None, :] * x
    np.testing.assert_allclose(y, expect, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("n", [32, 64])
def test_permuted_hadamard_closed_form(n):
    """S_U = P H (rows of H permuted by a cycle), S_V = H, l = c:
    W = c diag(h) P H H^T diag(g) = c n diag(h) P diag(g), so
    y_o = c n h_o g_pi(o) x_pi(o).  Pins that U's rows index the outputs and
    V's rows the inputs, and that h sits on the outputs and g on the inputs."""
    rng = np.random.default_rng(20 + n)
    H = sylvester(n)
    perm = np.roll(np.arange(n), 3)          # pi(o) = o - 3 mod n, not an involution
    su = H[perm]
    h = np.exp(rng.normal(-2, 0.5, n))
    g = np.exp(rng.normal(-2, 0.5, n))
    x = rng.standard_normal((2, n))
    c = 1.25
    y = oracle.forward(x, [dict(su=su, sv=H, h=h, g=g, l=np.full(n, c))])
    expect = c * n * h[None, :] * g[perm][None, :] * x[:, perm]
    np.testing.assert_allclose(y, expect, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("n,r", [(32, 8), (64, 16)])
def test_projector_closed_form(n, r):
    """S_U = S_V = H_n[:, :r] with unit scales gives W = P, P^2 = n P, rank r."""
    Hr = sylvester(n)[:, :r]
    ones = lambda k: np.ones(k)
    paths = [dict(su=Hr, sv=Hr, h=ones(n), g=ones(n), l=ones(r))]
    P = oracle.dense_weight(paths)
    assert np.array_equal(P @ P, n * P)
    assert np.linalg.matrix_rank(P) == r
    # forward on the identity returns W^T = P (P is symmetric)
    assert np.array_equal(oracle.forward(np.eye(n), paths), P.T)


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("seed", range(4))
def test_integer_exact_vs_brute_force(seed):
    """Unit scales and x in {-1, 0, 1}: every term is an integer, so the oracle
    and the brute-force sum agree exactly."""
    rng = np.random.default_rng(seed)
    n_in, n_out = int(rng.integers(5, 40)), int(rng.integers(3, 33))
    ranks = [int(rng.integers(1, 9)), int(rng.integers(1, 9))]
    x, paths = random_layer(rng, n_in, n_out, ranks, 3, unit_scales=True, int_x=True)
    y = oracle.forward(x, paths)
    assert np.array_equal(y, brute_force(x, paths))
    assert np.array_equal(y, np.rint(y))


@pytest.mark.parametrize("seed", range(4))
def test_random_vs_brute_force_and_dense(seed):
    rng = np.random.default_rng(100 + seed)
    n_in, n_out = int(rng.integers(4, 48)), int(rng.integers(4, 48))
    ranks = [int(rng.integers(1, 12))] + ([int(rng.integers(1, 12))] if seed % 2 else [])
    x, paths = random_layer(rng, n_in, n_out, ranks, 3)
    y = oracle.forward(x, paths)
    scale = np.abs(y).max()
    np.testing.assert_allclose(y, brute_force(x, paths), rtol=1e-12, atol=1e-12 * scale)
    np.testing.assert_allclose(y, x @ oracle.dense_weight(paths).T, rtol=1e-12,
                               atol=1e-12 * scale)


# ---------------------------------------------------------------- rank

@pytest.mark.parametrize("ranks", [[8], [5, 7], [3, 11]])
def test_numerical_rank(ranks):
    """rank(W) <= r (<= r1 + r2 with the residual), with equality for random
    signs at these sizes."""
    rng = np.random.default_rng(sum(ranks))
    _, paths = random_layer(rng, 48, 40, ranks, 1)
    W = oracle.dense_weight(paths)
    s = np.linalg.svd(W, compute_uv=False)
    rank = int(np.sum(s > 1e-9 * s[0]))
    assert rank == sum(ranks)


# ---------------------------------------------------------------- invariances

def test_sign_flip_pair_is_bitwise_invariant():
    rng = np.random.default_rng(7)
    x, paths = random_layer(rng, 64, 48, [16, 8], 4)
    y = oracle.forward(x, paths)
    flipped = [dict(p) for p in paths]
    for p in flipped:
        cols = rng.random(p["su"].shape[1]) < 0.5
        p["su"] = np.where(cols[None, :], -p["su"], p["su"]).astype(np.int8)
        p["sv"] = np.where(cols[None, :], -p["sv"], p["sv"]).astype(np.int8)
    assert np.array_equal(oracle.forward(x, flipped), y)


def test_joint_latent_permutation():
    rng = np.random.default_rng(8)
    x, paths = random_layer(rng, 64, 48, [16, 8], 4)
    y = oracle.forward(x, paths)
    permuted = []
    for p in paths:
        perm = rng.permutation(p["su"].shape[1])
        permuted.append(dict(p, su=p["su"][:, perm], sv=p["sv"][:, perm], l=p["l"][perm]))
    np.testing.assert_allclose(oracle.forward(x, permuted), y, rtol=1e-12,
                               atol=1e-12 * np.abs(y).max())


@pytest.mark.parametrize("alpha", [2.0, 0.25, 1024.0])
def test_power_of_two_rescale_is_bitwise(alpha):
    rng = np.random.default_rng(9)
    x, paths = random_layer(rng, 64, 48, [16, 8], 4)
    y = oracle.forward(x, paths)
    scaled = [dict(p, h=p["h"] * alpha, g=p["g"] / alpha) for p in paths]
    assert np.array_equal(oracle.forward(x, scaled), y)


# ---------------------------------------------------------------- mutations

def _pins_pass(fwd) -> bool:
    """Run the forward pins above against a (possibly mutated) forward
    function; True only if all of them hold."""
    fx = load_golden("forward_hand.txt")
    p1, p2 = hand_paths(fx)
    try:
        if not np.array_equal(fwd(np.array(fx["x"], float), [p1, p2]), np.array(fx["y"], float)):
            return False
        n = 32
        H = sylvester(n)
        perm = np.roll(np.arange(n), 3)
        rng = np.random.default_rng(0)
        h, g = np.exp(rng.normal(-2, .5, n)), np.exp(rng.normal(-2, .5, n))
        x = rng.standard_normal((2, n))
        y = fwd(x, [dict(su=H[perm], sv=H, h=h, g=g, l=np.full(n, 1.25))])
        if not np.allclose(y, 1.25 * n * h * g[perm] * x[:, perm], rtol=1e-12):
            return False
        x, paths = random_layer(np.random.default_rng(1), 12, 12, [3, 4], 2)
        if not np.allclose(fwd(x, paths), brute_force(x, paths), rtol=1e-12):
            return False
    except (ValueError, IndexError):
        return False          # a shape error is a caught mistake too
    return True


MUTANTS = {
    "drop_residual_path": lambda x, P: oracle.forward(x, P[:1]),
    "swap_h_and_g": lambda x, P: oracle.forward(
        x, [dict(p, h=p["g"], g=p["h"]) for p in P]),
    "swap_U_and_V": lambda x, P: oracle.forward(
        x, [dict(p, su=p["sv"], sv=p["su"]) for p in P]),
    "drop_latent_scale": lambda x, P: oracle.forward(
        x, [dict(p, l=np.ones(len(p["l"]))) for p in P]),
    "negate_one_factor": lambda x, P: oracle.forward(
        x, [dict(p, su=-np.asarray(p["su"], np.int8)) for p in P]),
    "reversed_input_index": lambda x, P: oracle.forward(
        x, [dict(p, sv=np.asarray(p["sv"], np.int8)[::-1]) for p in P]),
    "subtract_residual": lambda x, P: oracle.forward(x, P[:1]) - oracle.forward(x, P[1:]),
}


def test_unmutated_oracle_passes_pins():
    assert _pins_pass(oracle.forward)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name):
    assert not _pins_pass(MUTANTS[name]), f"mutant {name} slipped through the pins"


# ---------------------------------------------------------------- the two halves
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_latent_then_expand_is_forward_bitwise(seed):
    """expand(latent(x)) takes exactly the forward pass's steps in the same
    order, so it equals forward(x) bit for bit (the forward pass is pinned
    above)."""
    x, paths = random_layer(np.random.default_rng(40 + seed), 48, 40, [7, 12], 3)
    z = oracle.latent(x, paths)
    assert z.shape == (3, 19)
    assert np.array_equal(oracle.expand(z, paths), oracle.forward(x, paths))


def _exact_scales(rng, n):
    """Scales whose products are exact in fp64 (small binary fractions)."""
    return rng.choice([-2.0, -0.75, -0.5, 0.25, 0.5, 1.0, 1.5, 3.0], n)


def test_latent_closed_form_on_hadamard_columns():
    """V_sign = Sylvester H (rows i, columns k) and x = 2.5 e_j: the latent is
    z_k = l_k g_j 2.5 H[j, k], exactly; the second path (columns of H in
    reverse order) follows in the same row, after the first path's."""
    n = 32
    H = sylvester(n)
    rng = np.random.default_rng(7)
    p1 = dict(su=H, sv=H, h=_exact_scales(rng, n), g=_exact_scales(rng, n), l=_exact_scales(rng, n))
    p2 = dict(su=H[:, ::-1], sv=H[:, ::-1], h=_exact_scales(rng, n), g=_exact_scales(rng, n),
              l=_exact_scales(rng, n))
    for j in (0, 5, 31):
        x = np.zeros((1, n))
        x[0, j] = 2.5
        z = oracle.latent(x, [p1, p2])[0]
        assert np.array_equal(z[:n], p1["l"] * p1["g"][j] * 2.5 * H[j, :])
        assert np.array_equal(z[n:], p2["l"] * p2["g"][j] * 2.5 * H[j, ::-1])


def test_expand_closed_form_on_hadamard_rows():
    """U_sign = Sylvester H (rows o, columns k) and a latent 1.5 e_k in path 1
    and -0.5 e_k' in path 2: y_o = 1.5 h1_o H[o, k] - 0.5 h2_o H[o, k'], exactly."""
    n = 32
    H = sylvester(n)
    rng = np.random.default_rng(8)
    p1 = dict(su=H, sv=H, h=_exact_scales(rng, n), g=_exact_scales(rng, n), l=_exact_scales(rng, n))
    p2 = dict(su=H[::-1], sv=H, h=_exact_scales(rng, n), g=_exact_scales(rng, n), l=_exact_scales(rng, n))
    for k, k2 in ((0, 3), (17, 31)):
        z = np.zeros((1, 2 * n))
        z[0, k] = 1.5
        z[0, n + k2] = -0.5
        y = oracle.expand(z, [p1, p2])[0]
        assert np.array_equal(y, 1.5 * p1["h"] * H[:, k] + (-0.5) * p2["h"] * H[::-1][:, k2])
