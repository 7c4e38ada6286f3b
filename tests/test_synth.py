"""The seeded input generator: determinism, distributions, rounding, routing."""
import numpy as np
import pytest

import dbf_synth as S


def test_splitmix64_reference_words():
    # splitmix64 with state 0: the first outputs of the published generator
    # (Steele, Lea, Flood, "Fast splittable pseudorandom number generators", 2014)
    w = S.raw_u64(0, 3)
    assert [int(v) for v in w] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_streams_deterministic_and_distinct():
    a = S.raw_u64(S.stream_key(5, S.TAG_X), 100)
    b = S.raw_u64(S.stream_key(5, S.TAG_X), 100)
    c = S.raw_u64(S.stream_key(5, S.TAG_B1), 100)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)
    assert np.array_equal(S.raw_u64(S.stream_key(5, S.TAG_X), 50, offset=50), a[50:])


def test_normal_moments():
    v = S.normal(S.stream_key(1, 2), 200001)
    assert v.size == 200001
    assert abs(v.mean()) < 0.01 and abs(v.std() - 1.0) < 0.01


def test_signs_balanced_and_pm1():
    s = S.signs(S.stream_key(1, 3), 64, 1000)
    assert set(np.unique(s).tolist()) == {-1, 1}
    assert abs(s.astype(np.float64).mean()) < 0.01


def test_bf16_rounding_is_nearest_even():
    rng = np.random.default_rng(0)
    v = rng.standard_normal(5000).astype(np.float32)
    b = S.to_bf16_bits(v)
    got = S.bf16_bits_to_f32(b).astype(np.float64)
    # neighbours one bf16 ulp away are never closer
    up = S.bf16_bits_to_f32(b + 1).astype(np.float64)
    dn = S.bf16_bits_to_f32(b - 1).astype(np.float64)
    e = np.abs(got - v)
    assert np.all(e <= np.abs(up - v)) and np.all(e <= np.abs(dn - v))
    # exact ties go to the even pattern
    ties = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8], dtype=np.float32)
    tb = S.to_bf16_bits(ties)
    assert tb.tolist() == [0x3F80, 0x3F82]


def test_layer_shapes_and_scales():
    L = S.make_layer(9, 40, 24, 8, 2, 0.5)
    assert L.b1.shape == (24, 8) and L.b2.shape == (8, 40)
    assert L.alpha.shape == (2, 24) and L.beta.shape == (2, 8) and L.gamma.shape == (2, 40)
    a = L.alpha.view(np.float16).astype(np.float64)
    assert np.all(a > 0) and np.all(np.isfinite(a))


def test_segments_sorted_and_cover():
    seg = S.make_segments(77, 256, 32)
    assert seg.offsets[0] == 0 and seg.offsets[-1] == 256
    assert np.all(np.diff(seg.offsets) > 0)
    assert np.all(np.diff(seg.adapter) > 0) and seg.adapter.min() >= 0 and seg.adapter.max() < 32
    assert sorted(seg.order.tolist()) == list(range(256))


def test_sample_rows_holds_ends():
    r = S.sample_rows(3, 2048, 128)
    assert r.size == 128 and r[0] == 0 and r[-1] == 2047 and np.all(np.diff(r) > 0)


@pytest.mark.parametrize("T,n", [(2048, 128), (8192, 128), (2048, 64), (300, 2)])
def test_sample_rows_per_tile_covers_every_tile(T, n):
    r = S.sample_rows_per_tile(5, T, n, 256)
    assert r.size == n and r[0] == 0 and r[-1] == T - 1 and np.all(np.diff(r) > 0)
    tiles = (T + 255) // 256
    counts = np.bincount(r // 256, minlength=tiles)
    assert counts.min() >= n // tiles
    assert np.array_equal(r, S.sample_rows_per_tile(5, T, n, 256))


def test_weight_and_factor_start_recipes():
    # W[i, j] = g r_i c_j with lognormal row / column scales; seeded, distinct
    # streams for the weight and for the two start factors
    W1, W2 = S.make_weight(3, 64, 48), S.make_weight(3, 64, 48)
    assert W1.dtype == np.float32 and W1.shape == (64, 48) and np.array_equal(W1, W2)
    assert not np.array_equal(W1, S.make_weight(4, 64, 48))
    # row / column structure: the log of the row rms spreads with sigma 0.25
    big = S.make_weight(5, 2000, 2000).astype(np.float64)
    lr = np.log(np.sqrt((big ** 2).mean(axis=1)))
    assert 0.2 < lr.std() < 0.3
    U0, V0 = S.make_factor_start(6, 64, 48, 20, scale=2.0)
    assert U0.shape == (64, 20) and V0.shape == (20, 48) and U0.dtype == np.float32
    # U0 V0 entries have about the requested scale
    UV = U0.astype(np.float64) @ V0.astype(np.float64)
    assert 1.5 < np.sqrt((UV ** 2).mean()) < 2.6
