"""Pins of the fp64 oracle of the multi-boolean-kernel (MBOK) layer forward.

Multi-Boolean Architectures page, section 2: W ~ sum_k W_bool^[k] .
(s_out^[k] s_in^[k]^T), so y = W x with that W. Pinned by the dense
reconstruction with library matmuls, exact dyadic arithmetic (bit-identical),
the one-kernel all-ones case (a plain sign matrix product), additivity over
kernels, and per-kernel power-of-two scaling.
"""
import numpy as np
import pytest

import dbf_synth as S
import oracle
from test_oracle_pins import dec16, f16


def dense_w(L):
    w = np.zeros((L.N, L.M))
    for k in range(L.K):
        w += L.w[k].astype(np.float64) * np.outer(dec16(L.s_out[k]), dec16(L.s_in[k]))
    return w


def rand_layer(rng, M, N, K, dyadic=False):
    w = rng.choice(np.array([-1, 1], dtype=np.int8), size=(K, N, M))
    if dyadic:
        mk = lambda n: f16(rng.choice([0.5, 1.0, 2.0, -0.5, -2.0], n))
    else:
        mk = lambda n: f16(np.exp(0.5 * rng.standard_normal(n)) * rng.choice([-1.0, 1.0], n))
    return S.MbokLayer(M, N, K, w, np.stack([mk(M) for _ in range(K)]), np.stack([mk(N) for _ in range(K)]))


@pytest.mark.parametrize("M,N,K,T", [(7, 5, 1, 3), (9, 6, 2, 4), (16, 11, 4, 2)])
def test_dense_reconstruction(M, N, K, T):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    L = rand_layer(rng, M, N, K)
    x = rng.standard_normal((T, M)).astype(np.float32)
    np.testing.assert_allclose(oracle.mbok_forward(L, x), x.astype(np.float64) @ dense_w(L).T, rtol=1e-12, atol=1e-12)


def test_dyadic_bit_identical():
    rng = np.random.default_rng(5)
    L = rand_layer(rng, 12, 9, 3, dyadic=True)
    x = rng.integers(-2, 3, size=(4, 12)).astype(np.float32)
    assert np.array_equal(oracle.mbok_forward(L, x), x.astype(np.float64) @ dense_w(L).T)


def test_single_kernel_all_ones_is_a_sign_product():
    rng = np.random.default_rng(6)
    w = rng.choice(np.array([-1, 1], dtype=np.int8), size=(1, 8, 10))
    ones = lambda n: f16(np.ones(n))
    L = S.MbokLayer(10, 8, 1, w, ones(10)[None], ones(8)[None])
    x = rng.standard_normal((3, 10)).astype(np.float32)
    np.testing.assert_allclose(oracle.mbok_forward(L, x), x.astype(np.float64) @ w[0].T.astype(np.float64),
                               rtol=1e-13, atol=1e-13)


def test_additive_over_kernels_and_power_of_two_scaling():
    rng = np.random.default_rng(7)
    L = rand_layer(rng, 10, 7, 3)
    x = rng.standard_normal((2, 10)).astype(np.float32)
    parts = [oracle.mbok_forward(S.MbokLayer(10, 7, 1, L.w[k:k + 1], L.s_in[k:k + 1], L.s_out[k:k + 1]), x)
             for k in range(3)]
    np.testing.assert_allclose(oracle.mbok_forward(L, x), sum(parts), rtol=1e-12, atol=1e-12)
    so = L.s_out.copy()
    so[1] = f16(2 * dec16(so[1]))
    L2 = S.MbokLayer(10, 7, 3, L.w, L.s_in, so)
    np.testing.assert_allclose(oracle.mbok_forward(L2, x), parts[0] + 2 * parts[1] + parts[2], rtol=1e-12, atol=1e-12)


def test_synthetic_layer_shape_and_determinism():
    a = S.make_mbok_layer(0xDBF00006, 64, 32, 3)
    b = S.make_mbok_layer(0xDBF00006, 64, 32, 3)
    assert a.w.shape == (3, 32, 64) and a.s_in.shape == (3, 64) and a.s_out.shape == (3, 32)
    assert np.array_equal(a.w, b.w) and np.array_equal(a.s_in, b.s_in)
    assert set(np.unique(a.w)) <= {-1, 1}
