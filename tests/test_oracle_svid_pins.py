"""Pins of the oracle's SVID and successive MBOK extraction.

SVID (DBF page, section 2; Multi-Boolean Architectures page, section 2):
X ~ sign(X) . (s_out s_in^T) with the best rank-1 approximation of |X|.
Pinned by: exact recovery of a matrix whose magnitudes are rank one; sign
consistency; first-order optimality of the Frobenius error in s_out and
s_in (no gradient); the scaling law sqrt(c) per factor; and for successive
extraction, residual norms that never grow and reconstruction through the
oracle's MBOK forward.
"""
import numpy as np
import pytest

import dbf_synth as S
import oracle


def test_rank_one_magnitudes_are_recovered_exactly():
    rng = np.random.default_rng(1)
    p, q = rng.uniform(0.5, 2, 7), rng.uniform(0.5, 2, 5)
    sg = rng.choice([-1.0, 1.0], size=(7, 5))
    X = sg * np.outer(p, q)
    Sg, a, b = oracle.svid(X)
    np.testing.assert_array_equal(Sg, sg.astype(np.int8))
    np.testing.assert_allclose(Sg * np.outer(a, b), X, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("shape", [(6, 9), (13, 4), (32, 32)])
def test_first_order_optimality_and_signs(shape):
    rng = np.random.default_rng(shape[0] * 7 + shape[1])
    X = rng.standard_normal(shape)
    Sg, a, b = oracle.svid(X)
    assert np.array_equal(Sg, np.where(X < 0, -1, 1))
    assert np.all(a >= 0) and np.all(b >= 0)
    E = X - Sg * np.outer(a, b)
    # d/da ||E||^2 = -2 (E . S) b, d/db = -2 (E . S)^T a: both vanish at the optimum
    np.testing.assert_allclose((E * Sg) @ b, 0, atol=1e-10)
    np.testing.assert_allclose((E * Sg).T @ a, 0, atol=1e-10)
    # and no rank-one magnitude does better than it along random directions
    base = np.linalg.norm(E)
    for _ in range(5):
        da, db = rng.standard_normal(a.shape) * 1e-3, rng.standard_normal(b.shape) * 1e-3
        assert np.linalg.norm(X - Sg * np.outer(a + da, b + db)) >= base - 1e-12


def test_scaling_law():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((8, 6))
    _, a, b = oracle.svid(X)
    _, a4, b4 = oracle.svid(4.0 * X)
    np.testing.assert_allclose(a4, 2 * a, rtol=1e-12)
    np.testing.assert_allclose(b4, 2 * b, rtol=1e-12)


def test_successive_extraction_reconstructs_through_the_mbok_forward():
    rng = np.random.default_rng(4)
    W = rng.standard_normal((24, 40))
    w, so, si, norms = oracle.mbok_extract(W, 4)
    assert np.all(np.diff(norms) <= 1e-12)
    assert norms[-1] < norms[0]
    layer = S.MbokLayer(40, 24, 4, w, si, so)
    x = rng.standard_normal((3, 40)).astype(np.float32)
    y = oracle.mbok_forward(layer, x)
    W_hat = sum(w[k] * np.outer(so[k].view(np.float16).astype(np.float64), si[k].view(np.float16).astype(np.float64))
                for k in range(4))
    np.testing.assert_allclose(y, x.astype(np.float64) @ W_hat.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(W - W_hat), norms[-1], rtol=1e-12)
