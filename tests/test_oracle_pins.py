"""Pins of the fp64 oracle against facts other than itself.

Each check is chosen so that a plausible mistake in the oracle (a dropped
scale, an envelope index mixed up, a transposed factor, a wrong sign or
packed-bit position) fails at least one of them:

* dense reconstruction with library matmuls of the Delta-W equation of the
  LoRDBA page (section 2, "Arquitetura Central") and the DBF page (section 2),
  on random small shapes, M != N != R, ell up to 3, with and without
  accumulation;
* exact dyadic arithmetic: integer x and power-of-two scales make every
  partial sum exact, so oracle and dense results are bit-identical;
* closed forms: all signs +1, rank one, Sylvester-Hadamard factors;
* invariants: matched sign flips, envelope linearity, power-of-two scaling,
  permutation of the rank index;
* decoders against numpy's own fp16 / fp32 conversions over all patterns;
* the packed layout on hand-worked words (tests/golden/pack_layout.txt).
"""
import os

import numpy as np
import pytest

import dbf_synth as S
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f16(v):
    return np.asarray(v, dtype=np.float64).astype(np.float16).view(np.uint16)


def dec16(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def xval(x):
    if x.dtype == np.float32:
        return x.astype(np.float64)
    return S.bf16_bits_to_f32(x).astype(np.float64)


def dense_delta(L):
    """Delta-W = sum_i diag(alpha_i) B1 diag(beta_i) B2 diag(gamma_i), by matmul."""
    dw = np.zeros((L.N, L.M))
    b1 = L.b1.astype(np.float64)
    b2 = L.b2.astype(np.float64)
    for i in range(L.ell):
        dw += np.diag(dec16(L.alpha[i])) @ b1 @ np.diag(dec16(L.beta[i])) @ b2 @ np.diag(dec16(L.gamma[i]))
    return dw


def random_layer(rng, M, N, R, ell, scale_kind="lognormal"):
    b1 = rng.choice(np.array([-1, 1], dtype=np.int8), size=(N, R))
    b2 = rng.choice(np.array([-1, 1], dtype=np.int8), size=(R, M))
    if scale_kind == "lognormal":
        mk = lambda n: f16(np.exp(0.5 * rng.standard_normal(n)) * rng.choice([-1.0, 1.0], n))
    else:  # dyadic
        mk = lambda n: f16(rng.choice([0.5, 1.0, 2.0, -0.5, -1.0, -2.0], n))
    al = np.stack([mk(N) for _ in range(ell)])
    be = np.stack([mk(R) for _ in range(ell)])
    ga = np.stack([mk(M) for _ in range(ell)])
    return S.Layer(M, N, R, ell, b1, b2, al, be, ga)


def rel_err(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# ---------------------------------------------------------------- decoders

def test_f16_decoder_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_to_f64(bits)
    ref = bits.view(np.float16).astype(np.float64)
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert np.all(np.isnan(ours[~fin]))


def test_bf16_decoder_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    lib = oracle._load()
    ours = np.array([lib.dbf_oracle_bf16_to_f64(int(b)) for b in bits])
    ref = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert np.all(np.isnan(ours[~fin]))


def test_f32_decoder_samples():
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32)
    bits[:6] = [0, 0x80000000, 1, 0x007FFFFF, 0x7F7FFFFF, 0x3F800000]
    ours = oracle.f32_to_f64(bits)
    ref = bits.view(np.float32).astype(np.float64)
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])


# ------------------------------------------------------- dense reconstruction

@pytest.mark.parametrize("seed", range(8))
def test_matches_dense_reconstruction(seed):
    rng = np.random.default_rng(100 + seed)
    M, N, R = (int(v) for v in rng.integers(1, 64, size=3))
    ell = int(rng.integers(1, 4))
    L = random_layer(rng, M, N, R, ell)
    T = int(rng.integers(1, 6))
    x = rng.standard_normal((T, M)).astype(np.float32)
    acc = bool(seed % 2)
    y_in = rng.standard_normal((T, N)).astype(np.float32)
    got = oracle.forward(L, x, y_in=y_in, accumulate=acc)
    ref = x.astype(np.float64) @ dense_delta(L).T + (y_in.astype(np.float64) if acc else 0.0)
    assert rel_err(got, ref) < 1e-12


def test_tiny_workload_matches_dense():
    w = S.WORKLOADS["tiny"]
    L = S.workload_layers(w)[0]
    x = S.make_x(w.seed, 4, w.M, "f32")
    got = oracle.forward(L, x)
    ref = x.astype(np.float64) @ dense_delta(L).T
    assert rel_err(got, ref) < 1e-12


def test_bf16_activations_and_row_subset():
    rng = np.random.default_rng(3)
    L = random_layer(rng, 40, 24, 12, 2)
    xb = S.to_bf16_bits(rng.standard_normal((7, 40)))
    rows = [6, 0, 3]
    got = oracle.forward(L, xb, rows=rows)
    ref = xval(xb)[rows] @ dense_delta(L).T
    assert rel_err(got, ref) < 1e-12


@pytest.mark.parametrize("seed", range(4))
def test_exact_dyadic_bit_identical(seed):
    # integer x in [-2, 2], scales in {+-1/2, +-1, +-2}: every partial sum is a
    # small dyadic rational, exact in fp64 in any order
    rng = np.random.default_rng(200 + seed)
    M, N, R = 48, 40, 24
    L = random_layer(rng, M, N, R, 1 + seed % 3, scale_kind="dyadic")
    x = rng.integers(-2, 3, size=(5, M)).astype(np.float32)
    got = oracle.forward(L, x)
    ref = x.astype(np.float64) @ dense_delta(L).T
    assert np.array_equal(got, ref)


# ------------------------------------------------------------- closed forms

def test_closed_form_all_plus():
    rng = np.random.default_rng(11)
    M, N, R, ell = 33, 21, 17, 2
    L = random_layer(rng, M, N, R, ell)
    L.b1[:] = 1
    L.b2[:] = 1
    x = rng.standard_normal((3, M)).astype(np.float32)
    got = oracle.forward(L, x)
    ref = np.zeros((3, N))
    for i in range(ell):
        a, b, g = dec16(L.alpha[i]), dec16(L.beta[i]), dec16(L.gamma[i])
        ref += np.outer((x.astype(np.float64) * g).sum(axis=1) * b.sum(), a)
    assert rel_err(got, ref) < 1e-12


def test_closed_form_rank_one():
    rng = np.random.default_rng(12)
    M, N, ell = 50, 30, 2
    L = random_layer(rng, M, N, 1, ell)
    x = rng.standard_normal((4, M)).astype(np.float32)
    got = oracle.forward(L, x)
    ref = np.zeros((4, N))
    for i in range(ell):
        a, b, g = dec16(L.alpha[i]), dec16(L.beta[i])[0], dec16(L.gamma[i])
        s = (x.astype(np.float64) * g) @ L.b2[0].astype(np.float64)      # b2^T (gamma . x)
        ref += np.outer(s * b, a * L.b1[:, 0])
    assert rel_err(got, ref) < 1e-12


def sylvester(n):
    h = np.array([[1]], dtype=np.int8)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]]).astype(np.int8)
    return h


@pytest.mark.parametrize("n", [1, 2, 8, 64])
def test_closed_form_hadamard(n):
    # B1 = B2 = H_n (symmetric, H H = n I), beta = c: y = c n (alpha . gamma . x)
    rng = np.random.default_rng(13)
    L = random_layer(rng, n, n, n, 1)
    H = sylvester(n)
    L.b1[:] = H
    L.b2[:] = H
    c = 0.75
    L.beta[:] = f16(np.full(n, c))
    x = rng.standard_normal((3, n)).astype(np.float32)
    got = oracle.forward(L, x)
    ref = c * n * dec16(L.alpha[0]) * dec16(L.gamma[0]) * x.astype(np.float64)
    assert rel_err(got, ref) < 1e-12


# --------------------------------------------------------------- invariants

def test_matched_sign_flip_bit_identical():
    rng = np.random.default_rng(21)
    L = random_layer(rng, 45, 37, 19, 2)
    x = rng.standard_normal((4, 45)).astype(np.float32)
    y0 = oracle.forward(L, x)
    flip = rng.random(19) < 0.5
    L.b1[:, flip] *= -1
    L.b2[flip, :] *= -1
    y1 = oracle.forward(L, x)
    assert np.array_equal(y0, y1)


def test_unmatched_flip_changes_result():
    rng = np.random.default_rng(22)
    L = random_layer(rng, 45, 37, 19, 1)
    x = rng.standard_normal((2, 45)).astype(np.float32)
    y0 = oracle.forward(L, x)
    L.b2[3, :] *= -1            # flip only the B2 row
    assert rel_err(oracle.forward(L, x), y0) > 1e-3


def test_envelope_linearity():
    rng = np.random.default_rng(23)
    L = random_layer(rng, 30, 26, 14, 2)
    x = rng.standard_normal((3, 30)).astype(np.float32)
    y2 = oracle.forward(L, x)
    parts = []
    for i in range(2):
        Li = S.Layer(L.M, L.N, L.R, 1, L.b1, L.b2, L.alpha[i:i + 1], L.beta[i:i + 1], L.gamma[i:i + 1])
        parts.append(oracle.forward(Li, x))
    assert rel_err(y2, parts[0] + parts[1]) < 1e-12


def test_power_of_two_alpha_scaling_exact():
    rng = np.random.default_rng(24)
    L = random_layer(rng, 30, 26, 14, 1)
    x = rng.standard_normal((3, 30)).astype(np.float32)
    y0 = oracle.forward(L, x)
    L.alpha[:] = f16(2.0 * dec16(L.alpha))
    assert np.array_equal(oracle.forward(L, x), 2.0 * y0)


def test_rank_permutation():
    rng = np.random.default_rng(25)
    L = random_layer(rng, 30, 26, 14, 2)
    x = rng.standard_normal((3, 30)).astype(np.float32)
    y0 = oracle.forward(L, x)
    p = rng.permutation(14)
    Lp = S.Layer(L.M, L.N, L.R, L.ell, L.b1[:, p], L.b2[p, :], L.alpha, L.beta[:, p], L.gamma)
    assert rel_err(oracle.forward(Lp, x), y0) < 1e-12


def test_rank_permutation_without_beta_breaks():
    # permuting B1 / B2 but not beta must change the result (beta is indexed by r)
    rng = np.random.default_rng(26)
    L = random_layer(rng, 30, 26, 14, 1)
    x = rng.standard_normal((3, 30)).astype(np.float32)
    y0 = oracle.forward(L, x)
    p = np.roll(np.arange(14), 1)
    Lp = S.Layer(L.M, L.N, L.R, L.ell, L.b1[:, p], L.b2[p, :], L.alpha, L.beta, L.gamma)
    assert rel_err(oracle.forward(Lp, x), y0) > 1e-3


# ----------------------------------------------------------------- segments

def test_segmented_matches_per_token_dense():
    rng = np.random.default_rng(31)
    M, N, R, ell = 20, 18, 6, 2
    layers = [random_layer(rng, M, N, R, ell) for _ in range(3)]
    T = 11
    x = rng.standard_normal((T, M)).astype(np.float32)
    y_in = rng.standard_normal((T, N)).astype(np.float32)
    offsets = [0, 3, 3, 7, 9, 11]           # includes an empty segment
    adapter = [2, 0, 1, -1, 0]               # and a token range with no adapter
    for acc in (False, True):
        got = oracle.forward_segmented(layers, offsets, adapter, x, y_in=y_in, accumulate=acc)
        ref = np.zeros((T, N))
        for s, a in enumerate(adapter):
            for t in range(offsets[s], offsets[s + 1]):
                base = y_in[t].astype(np.float64) if acc else 0.0
                ref[t] = base + (dense_delta(layers[a]) @ x[t].astype(np.float64) if a >= 0 else 0.0)
        assert rel_err(got, ref) < 1e-12


# ------------------------------------------------------------------ packing

def read_golden():
    cases = []
    with open(os.path.join(GOLDEN, "pack_layout.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, cols, words = (p.strip() for p in line.split("|"))
            cases.append((int(k), cols, [int(w, 16) for w in words.split(",")]))
    return cases


@pytest.mark.parametrize("case", read_golden(), ids=lambda c: f"k{c[0]}-{c[1]}")
def test_pack_golden_words(case):
    k, cols, words = case
    s = np.ones((1, k), dtype=np.int8)
    if cols == "all":
        s[:] = -1
    elif cols != "none":
        for c in cols.split(","):
            s[0, int(c)] = -1
    got = oracle.pack(s)
    assert got.tolist() == [words]
    assert np.array_equal(oracle.unpack(got, 1, k), s)


@pytest.mark.parametrize("shape", [(1, 1), (3, 31), (5, 32), (4, 33), (7, 100), (16, 5888 // 23)])
def test_pack_roundtrip_and_padding(shape):
    rows, k = shape
    rng = np.random.default_rng(rows * 1000 + k)
    s = rng.choice(np.array([-1, 1], dtype=np.int8), size=shape)
    w = oracle.pack(s)
    assert w.shape == (rows, (k + 31) // 32)
    assert np.array_equal(oracle.unpack(w, rows, k), s)
    # padding bits past k are zero: pack of all -1 sets exactly k bits per row
    wa = oracle.pack(-np.ones(shape, dtype=np.int8))
    pop = np.array([[bin(int(v)).count("1") for v in row] for row in wa]).sum(axis=1)
    assert np.all(pop == k)


def test_latent_sign_convention():
    h = np.array([-1.5, -0.0, 0.0, 2.0, -1e-30, 1e-30])
    assert oracle.sign_of_latent(h).tolist() == [-1, 1, 1, 1, -1, 1]
    with pytest.raises(ValueError):
        oracle.sign_of_latent(np.array([1.0, np.nan]))
