"""Pins of the fp64 oracle backward against facts other than itself.

The backward (gradients of L = sum dy . y through the forward of the LoRDBA
page, section 2) is pinned only through the *forward* oracle, which the
forward pins tie to the Delta-W equation, and through linear algebra:

* y is linear in every single parameter entry (a scale entry, an input
  entry, one sign entry taken as a real number), so setting one entry to
  zero, or negating one sign, changes L by exactly -entry * gradient or
  -2 * sign * gradient: difference quotients with no step-size error;
* Euler's identity for functions of degree one: sum(theta . dL/dtheta) = L
  for each of alpha, beta, gamma, x, B1, B2 taken as a whole;
* dx = dy Delta-W with Delta-W reconstructed by library matmuls;
* bf16 inputs give the same gradients as their exact fp32 values.

A dropped scale, a transposed factor, a wrong envelope index or a sign slip
in any gradient fails at least one of these.
"""
import numpy as np
import pytest

import dbf_synth as S
import oracle
from test_oracle_pins import dec16, dense_delta, random_layer

SHAPES = [(7, 5, 6, 1, 3), (6, 9, 4, 2, 2), (5, 4, 8, 3, 4)]   # M, N, R, ell, T


def loss(L, x, dy):
    return float((oracle.forward(L, x) * dy.astype(np.float64)).sum())


def with_field(L, **kw):
    d = dict(M=L.M, N=L.N, R=L.R, ell=L.ell, b1=L.b1, b2=L.b2, alpha=L.alpha, beta=L.beta, gamma=L.gamma)
    d.update(kw)
    return S.Layer(**d)


@pytest.fixture(params=SHAPES, ids=lambda s: "M{}N{}R{}l{}T{}".format(*s))
def case(request):
    M, N, R, ell, T = request.param
    rng = np.random.default_rng(1000 + M * 7 + N * 3 + R + ell + T)
    L = random_layer(rng, M, N, R, ell)
    x = rng.standard_normal((T, M)).astype(np.float32)
    dy = rng.standard_normal((T, N)).astype(np.float32)
    return L, x, dy, oracle.backward(L, x, dy, want_signs=True)


def test_scale_gradients_by_zeroing_one_entry(case):
    L, x, dy, g = case
    L0 = loss(L, x, dy)
    for name, grad in (("alpha", g.dalpha), ("beta", g.dbeta), ("gamma", g.dgamma)):
        bits = getattr(L, name)
        for i in range(L.ell):
            for k in range(bits.shape[1]):
                val = dec16(bits[i, k])
                b = bits.copy()
                b[i, k] = 0
                d = L0 - loss(with_field(L, **{name: b}), x, dy)
                assert d == pytest.approx(val * grad[i, k], rel=1e-9, abs=1e-9), (name, i, k)


def test_input_gradient_by_zeroing_one_entry(case):
    L, x, dy, g = case
    L0 = loss(L, x, dy)
    for t in range(x.shape[0]):
        for m in range(L.M):
            x2 = x.copy()
            x2[t, m] = 0.0
            d = L0 - loss(L, x2, dy)
            assert d == pytest.approx(float(x[t, m]) * g.dx[t, m], rel=1e-9, abs=1e-9)


def test_sign_gradients_by_flipping_one_sign(case):
    L, x, dy, g = case
    L0 = loss(L, x, dy)
    for name, grad in (("b1", g.db1), ("b2", g.db2)):
        B = getattr(L, name)
        for idx in np.ndindex(*B.shape):
            B2 = B.copy()
            B2[idx] = -B2[idx]
            d = loss(with_field(L, **{name: B2}), x, dy) - L0
            assert d == pytest.approx(-2.0 * B[idx] * grad[idx], rel=1e-9, abs=1e-9), (name, idx)


def test_euler_identity(case):
    L, x, dy, g = case
    L0 = loss(L, x, dy)
    assert (dec16(L.alpha) * g.dalpha).sum() == pytest.approx(L0, rel=1e-12, abs=1e-12)
    assert (dec16(L.beta) * g.dbeta).sum() == pytest.approx(L0, rel=1e-12, abs=1e-12)
    assert (dec16(L.gamma) * g.dgamma).sum() == pytest.approx(L0, rel=1e-12, abs=1e-12)
    assert (x.astype(np.float64) * g.dx).sum() == pytest.approx(L0, rel=1e-12, abs=1e-12)
    # degree one in B1 (and in B2) for each envelope, so also as a whole
    assert (L.b1 * g.db1).sum() == pytest.approx(L0, rel=1e-12, abs=1e-12)
    assert (L.b2 * g.db2).sum() == pytest.approx(L0, rel=1e-12, abs=1e-12)


def test_input_gradient_is_transposed_dense_product(case):
    L, x, dy, g = case
    ref = dy.astype(np.float64) @ dense_delta(L)
    np.testing.assert_allclose(g.dx, ref, rtol=1e-12, atol=1e-12)


def test_bf16_inputs_match_their_fp32_values():
    rng = np.random.default_rng(77)
    L = random_layer(rng, 9, 6, 5, 2)
    xb = S.to_bf16_bits(rng.standard_normal((3, 9)))
    db = S.to_bf16_bits(rng.standard_normal((3, 6)))
    gb = oracle.backward(L, xb, db, want_signs=True)
    gf = oracle.backward(L, S.bf16_bits_to_f32(xb), S.bf16_bits_to_f32(db), want_signs=True)
    for a, b in ((gb.dx, gf.dx), (gb.dalpha, gf.dalpha), (gb.dbeta, gf.dbeta), (gb.dgamma, gf.dgamma),
                 (gb.db1, gf.db1), (gb.db2, gf.db2)):
        assert np.array_equal(a, b)


def test_thread_split_does_not_change_results():
    rng = np.random.default_rng(78)
    L = random_layer(rng, 8, 7, 6, 2)
    x = rng.standard_normal((9, 8)).astype(np.float32)
    dy = rng.standard_normal((9, 7)).astype(np.float32)
    g1 = oracle.backward(L, x, dy, want_signs=True, nthreads=1)
    g4 = oracle.backward(L, x, dy, want_signs=True, nthreads=4)
    np.testing.assert_allclose(g4.dalpha, g1.dalpha, rtol=1e-13)
    np.testing.assert_array_equal(g4.dx, g1.dx)


@pytest.mark.parametrize("tau", [0.25, 1.0, 3.0])
def test_ste_surrogate_derivative_matches_the_surrogate(tau):
    # the derivative the oracle uses against a central difference of tanh(h/tau)
    h = np.linspace(-4, 4, 97)
    eps = 1e-6
    fd = (np.tanh((h + eps) / tau) - np.tanh((h - eps) / tau)) / (2 * eps)
    np.testing.assert_allclose(oracle.ste_backward(np.ones_like(h), h, tau), fd, rtol=1e-7, atol=1e-9)
    # slope 1/tau at zero, odd-symmetric surrogate -> even derivative
    assert oracle.ste_backward(np.array([2.0]), np.array([0.0]), tau)[0] == pytest.approx(2.0 / tau)


def test_ste_clipped_identity():
    h = np.array([-1.5, -1.0, -0.3, 0.0, 0.999, 1.0, 1.0001, 7.0])
    db = np.arange(1, 9, dtype=np.float64)
    np.testing.assert_array_equal(oracle.ste_backward(db, h, 0.0), db * np.array([0, 1, 1, 1, 1, 1, 0, 0]))
