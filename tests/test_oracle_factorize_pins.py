"""Pins of the oracle's DBF factorisation (DBF page, section 2: alternating
minimisation with ADMM and the SVID projection) against facts that do not
come from the oracle itself:

- each least-squares step satisfies the first-order condition of the
  objective it minimises (gradient computed here from the objective);
- the exact product of two members of the constraint set, used as the start,
  is a fixed point of the whole iteration;
- at k = 1 every column / row vector lies in the constraint set, so the
  iteration is alternating least squares for a rank-1 fit and must reach the
  Eckart-Young error sqrt(|W|^2 - sigma_1^2) (sigma_1 from numpy's SVD);
- the returned signs and fp16 scales, run through the layer forward (the
  oracle's C forward, pinned on its own), reproduce the product they define.
"""
import numpy as np
import pytest

import dbf_synth as S
import oracle
from oracle import admm_u_step, admm_v_step, factorize, svd_init


def weight(seed, n, m):
    """A weight with row and column scale structure (lognormal 0.25)."""
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((n, m)) * np.exp(0.25 * rng.standard_normal(n))[:, None]
            * np.exp(0.25 * rng.standard_normal(m))[None, :])


def member(rng, r, c):
    """A random member of the constraint set: diag(p) S diag(q), p, q > 0."""
    Sg = rng.choice([-1.0, 1.0], size=(r, c))
    return np.exp(0.3 * rng.standard_normal(r))[:, None] * Sg * np.exp(0.3 * rng.standard_normal(c))[None, :]


def test_u_step_first_order_condition():
    rng = np.random.default_rng(1)
    n, m, k = 30, 25, 12
    W, V = rng.standard_normal((n, m)), rng.standard_normal((k, m))
    Z, Lam, rho = rng.standard_normal((n, k)), rng.standard_normal((n, k)), 0.7
    U = admm_u_step(W @ V.T, V @ V.T, rho, Z, Lam)
    grad = -(W - U @ V) @ V.T + rho * (U - Z + Lam)
    assert np.abs(grad).max() <= 1e-10 * np.abs(W @ V.T).max()


def test_v_step_first_order_condition():
    rng = np.random.default_rng(2)
    n, m, k = 30, 25, 12
    W, U = rng.standard_normal((n, m)), rng.standard_normal((n, k))
    Z, Lam, rho = rng.standard_normal((k, m)), rng.standard_normal((k, m)), 1.3
    V = admm_v_step(U.T @ W, U.T @ U, rho, Z, Lam)
    grad = -U.T @ (W - U @ V) + rho * (V - Z + Lam)
    assert np.abs(grad).max() <= 1e-10 * np.abs(U.T @ W).max()


@pytest.mark.parametrize("n,m,k", [(40, 30, 8), (24, 56, 32)])
def test_exact_product_is_a_fixed_point(n, m, k):
    rng = np.random.default_rng(n + m + k)
    Ut, Vt = member(rng, n, k), member(rng, k, m)
    W = Ut @ Vt
    f = factorize(W, Ut, Vt, outer=3, admm_iters=3)
    assert max(f.objective) <= 1e-10 * np.linalg.norm(W)
    np.testing.assert_allclose(f.U, Ut, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(f.V, Vt, rtol=1e-10, atol=1e-12)
    assert np.array_equal(f.A, np.sign(Ut)) and np.array_equal(f.B, np.sign(Vt))


def test_rank_one_reaches_eckart_young():
    rng = np.random.default_rng(3)
    n, m = 30, 20
    W = 4.0 * np.outer(rng.standard_normal(n), rng.standard_normal(m)) + rng.standard_normal((n, m))
    U0, V0 = rng.standard_normal((n, 1)), rng.standard_normal((1, m))
    f = factorize(W, U0, V0, outer=60, admm_iters=3)
    s = np.linalg.svd(W, compute_uv=False)
    best = np.sqrt(np.sum(s[1:] ** 2))
    assert abs(f.objective[-1] - best) <= 1e-9 * np.linalg.norm(W)
    assert f.objective[0] > best * 1.01   # the start is not already optimal


def test_layer_forward_reproduces_the_factors():
    W = weight(4, 48, 40)
    U0, V0 = svd_init(W, 20)
    f = factorize(W, U0, V0, outer=3, admm_iters=3)
    L = f.layer()
    dec = lambda bits: bits.astype(np.uint16).view(np.float16).astype(np.float64)
    What = (dec(f.alpha)[:, None] * f.A) @ (dec(f.beta)[:, None] * f.B) * dec(f.gamma)[None, :]
    x = np.random.default_rng(5).standard_normal((7, 40)).astype(np.float32)
    y = oracle.forward(L, x)
    np.testing.assert_allclose(y, x.astype(np.float64) @ What.T, rtol=1e-12, atol=1e-12)
    # fp16 rounding of the scales moves the product by a few 1e-4 at most
    assert np.abs(What - f.U @ f.V).max() <= 2e-3 * np.abs(f.U @ f.V).max()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_objective_falls_from_the_projected_start(seed):
    # a seeded property, not a theorem: the scheme is a heuristic
    W = weight(10 + seed, 64, 48)
    U0, V0 = svd_init(W, 24)
    f = factorize(W, U0, V0, outer=6, admm_iters=4)
    o = np.array(f.objective)
    assert np.all(np.isfinite(o))
    assert o[-1] < 0.95 * o[0]
    assert np.all(np.diff(o) <= 1e-3 * o[0])


def test_svd_init_is_the_truncated_svd():
    W = weight(6, 30, 22)
    U0, V0 = svd_init(W, 7)
    s = np.linalg.svd(W, compute_uv=False)
    assert abs(np.linalg.norm(W - U0 @ V0) - np.sqrt(np.sum(s[7:] ** 2))) <= 1e-10 * np.linalg.norm(W)
