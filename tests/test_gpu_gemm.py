"""The tcgen05 prefill path (DBF_PATH_GEMM) against the fp64 oracle.

The GEMM rounds gamma.x and beta.h to fp16 operands and accumulates in fp32,
so its error is a few 1e-4 of max|y|, inside the 2e-3 contract. Integer
inputs chosen so that every fp16 operand and fp32 sum is exact must give
bit-identical results: that pins the shared-memory layouts, descriptors,
tile indexing and the alpha fold independently of rounding.
"""
import numpy as np
import pytest
import torch

import dbf_synth as S
import oracle
from gpu_util import TOL, bf16_ok, dev_layer, dev_x, host_y, random_layer, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbf():
    import double_binary_rank_b200 as m
    return m


def run(dbf, L, x, y_dtype=torch.float32, acc=False, y_in=None, path="gemm"):
    dl = dev_layer(L)
    y = torch.from_numpy(y_in).cuda().to(y_dtype) if acc else None
    out = dbf.forward(dl, dev_x(x), y=y, accumulate=acc, path=path, y_dtype=y_dtype)
    torch.cuda.synchronize()
    return host_y(out)


def exact_layer(rng, M, N, R, ell):
    b1 = rng.choice(np.array([-1, 1], dtype=np.int8), size=(N, R))
    b2 = rng.choice(np.array([-1, 1], dtype=np.int8), size=(R, M))
    f = lambda vals, n: S.to_f16_bits(rng.choice(vals, n))
    return S.Layer(M, N, R, ell, b1, b2,
                   np.stack([f([0.5, 1.0, 2.0, -0.5, -1.0, -2.0], N) for _ in range(ell)]),
                   np.stack([f([1.0, 2.0, -1.0, -2.0], R) for _ in range(ell)]),
                   np.stack([f([1.0, -1.0], M) for _ in range(ell)]))


@pytest.mark.parametrize("shape", [(128, 16, 128, 1, 1), (256, 200, 128, 1, 7), (128, 136, 256, 2, 300),
                                   (384, 64, 128, 3, 33)], ids=lambda s: "M{}N{}R{}l{}T{}".format(*s))
def test_gemm_exact_bit_identical(dbf, shape):
    M, N, R, ell, T = shape
    rng = np.random.default_rng(sum(shape))
    L = exact_layer(rng, M, N, R, ell)
    x = rng.integers(-1, 2, size=(T, M)).astype(np.float32)
    ref = oracle.forward(L, x)
    got = run(dbf, L, x)
    assert np.array_equal(got, ref), float(np.max(np.abs(got - ref)))


# M = 1152: the pre-pass converts rows in 1024-column pieces, the last one
# partial
@pytest.mark.parametrize("shape", [(128, 48, 128, 1, 5), (512, 300, 384, 2, 260), (256, 1024, 256, 1, 513),
                                   (1152, 200, 256, 2, 37)],
                         ids=lambda s: "M{}N{}R{}l{}T{}".format(*s))
@pytest.mark.parametrize("acc", [False, True])
def test_gemm_random(dbf, shape, acc):
    M, N, R, ell, T = shape
    rng = np.random.default_rng(sum(shape) + 7)
    L = random_layer(rng, M, N, R, ell)
    x = S.to_bf16_bits(rng.standard_normal((T, M)))
    y_in = rng.standard_normal((T, N)).astype(np.float32)
    ref = oracle.forward(L, x, y_in=y_in, accumulate=acc)
    got = run(dbf, L, x, acc=acc, y_in=y_in)
    assert rel_err(got, ref) < TOL


def test_gemm_matches_gemv(dbf):
    rng = np.random.default_rng(70)
    L = random_layer(rng, 256, 160, 128, 2)
    x = S.to_bf16_bits(rng.standard_normal((40, 256)))
    a = run(dbf, L, x, path="gemm")
    b = run(dbf, L, x, path="gemv")
    assert rel_err(a, b) < TOL


def check_rows_cover_tiles(rows, T, tile=256):
    """The sampled rows include the first and the last token and at least one
    row of every 256-token tile of the GEMM, so that every tile the
    persistent schedule hands out (including those past the first wave of
    148) is checked."""
    assert rows[0] == 0 and rows[-1] == T - 1
    assert set(range((T + tile - 1) // tile)) <= set(int(r) // tile for r in rows)


def test_dbf_mlp_prefill_sampled_rows(dbf):
    # the DBF MLP layer at 2048 tokens, checked on a fixed sample of 128 token rows
    w = S.WORKLOADS["dbf_mlp"]
    L = S.workload_layers(w)[0]
    T = 2048
    x = S.make_x(w.seed, T, w.M, "bf16")
    rows = S.sample_rows_per_tile(w.seed, T, 128, 256)
    assert len(rows) == 128
    check_rows_cover_tiles(rows, T)
    ref = oracle.forward(L, x, rows=rows)
    got = run(dbf, L, x, y_dtype=torch.float32)[rows]
    assert rel_err(got, ref) < TOL
    got_b = run(dbf, L, x, y_dtype=torch.bfloat16)[rows]
    ok, worst = bf16_ok(got_b, ref)
    assert ok, worst


def test_dbf_mlp_prefill_deterministic(dbf):
    # The DBF MLP layer at 2048 tokens takes the one-launch forward with its
    # last stage-2 tiles split in K: which pair runs which tile, and which half
    # of a split tile finishes first, vary between calls; y does not.
    w = S.WORKLOADS["dbf_mlp"]
    L = S.workload_layers(w)[0]
    x = S.make_x(w.seed + 7, 2048, w.M, "bf16")
    dl = dev_layer(L)
    xd = dev_x(x)
    a = dbf.forward(dl, xd, path="gemm", y_dtype=torch.float32)
    b = dbf.forward(dl, xd, path="gemm", y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_large_prefill_sampled_rows(dbf):
    # M = N = R = 8192 at 8192 tokens, checked on a fixed sample of token rows
    w = S.WORKLOADS["large_prefill"]
    L = S.workload_layers(w)[0]
    T = 8192
    x = S.make_x(w.seed, T, w.M, "bf16")
    rows = S.sample_rows_per_tile(w.seed, T, 128, 256)
    assert len(rows) == 128
    check_rows_cover_tiles(rows, T)
    ref = oracle.forward(L, x, rows=rows)
    got = run(dbf, L, x, y_dtype=torch.float32)[rows]
    assert rel_err(got, ref) < TOL


# Shape whose two GEMM stages each have 256 tiles (32 row tiles x 8 token
# tiles), so the persistent kernel's CTAs wrap past the first 148 tiles.
WRAP = dict(M=1024, N=4096, R=4096, T=2048)


def test_gemm_matched_sign_flip_bit_identical(dbf):
    # Negating column r of B1 and row r of B2 negates h_r and v_r exactly
    # (round to nearest even is symmetric) and leaves every product of stage
    # 2 unchanged, so with a fixed accumulation order y is bit-identical.
    rng = np.random.default_rng(60)
    L = random_layer(rng, WRAP["M"], WRAP["N"], WRAP["R"], 1)
    x = S.to_bf16_bits(rng.standard_normal((WRAP["T"], WRAP["M"])))
    y0 = run(dbf, L, x)
    flip = rng.random(WRAP["R"]) < 0.5
    L.b1[:, flip] *= -1
    L.b2[flip, :] *= -1
    y1 = run(dbf, L, x)
    assert np.array_equal(y0, y1)


def test_gemm_power_of_two_alpha_bit_exact(dbf):
    # alpha -> 2 alpha doubles the fp16 A operand exactly, and scaling by two
    # commutes with every fp32 rounding: y -> exactly 2 y.
    rng = np.random.default_rng(61)
    L = random_layer(rng, WRAP["M"], WRAP["N"], WRAP["R"], 1)
    x = S.to_bf16_bits(rng.standard_normal((WRAP["T"], WRAP["M"])))
    y0 = run(dbf, L, x)
    L.alpha[:] = S.to_f16_bits(2.0 * L.alpha.view(np.float16).astype(np.float64))
    y1 = run(dbf, L, x)
    assert np.array_equal(y1, 2.0 * y0)


def test_gemm_wrapping_shape_sampled_rows(dbf):
    # the same shape against the oracle on rows of every token tile
    rng = np.random.default_rng(62)
    L = random_layer(rng, WRAP["M"], WRAP["N"], WRAP["R"], 1)
    T = WRAP["T"]
    x = S.to_bf16_bits(rng.standard_normal((T, WRAP["M"])))
    rows = S.sample_rows_per_tile(62, T, 64, 256)
    check_rows_cover_tiles(rows, T)
    ref = oracle.forward(L, x, rows=rows)
    got = run(dbf, L, x)[rows]
    assert rel_err(got, ref) < TOL


# Shapes that take the single-launch forward (both stages at least 32 K steps
# deep): tiles claimed at run time, stage-2 tiles that wait for the stage-1
# column blocks they read, ragged rows and tokens; the second has two
# envelopes whose column blocks straddle the envelope boundary (ell T = 2200),
# the second and third split their last stage-2 tiles in K, and the last two
# have one and three tokens (one column block).
FUSED = [(2048, 1000, 2048, 1, 700), (2048, 2500, 1024, 2, 1100), (4096, 4096, 2048, 1, 1024),
         (2048, 512, 2048, 1, 1), (2048, 768, 1024, 2, 3), (2176, 640, 2048, 1, 300)]


@pytest.mark.parametrize("shape", FUSED, ids=lambda s: "M{}N{}R{}l{}T{}".format(*s))
def test_fused_forward_against_oracle(dbf, shape):
    M, N, R, ell, T = shape
    rng = np.random.default_rng(sum(shape) + 11)
    L = random_layer(rng, M, N, R, ell)
    x = S.to_bf16_bits(rng.standard_normal((T, M)))
    y_in = rng.standard_normal((T, N)).astype(np.float32)
    ref = oracle.forward(L, x)
    got = run(dbf, L, x)
    assert rel_err(got, ref) < TOL
    ref_acc = oracle.forward(L, x, y_in=y_in, accumulate=True)
    assert rel_err(run(dbf, L, x, acc=True, y_in=y_in), ref_acc) < TOL
    ok, worst = bf16_ok(run(dbf, L, x, y_dtype=torch.bfloat16), ref)
    assert ok, worst


def test_fused_forward_deterministic_and_exact(dbf):
    # Which pair computes a tile depends on timing, its accumulation order
    # does not: two calls agree bit for bit. Integer inputs with exact fp16
    # operands and fp32 sums match the oracle exactly.
    M, N, R, ell, T = 2048, 2500, 1024, 2, 1100
    rng = np.random.default_rng(63)
    L = exact_layer(rng, M, N, R, ell)
    x = rng.integers(-1, 2, size=(T, M)).astype(np.float32)
    a = run(dbf, L, x)
    b = run(dbf, L, x)
    assert np.array_equal(a, b)
    assert np.array_equal(a, oracle.forward(L, x))


# shapes whose schedule on 74 CTA pairs (a full B200) splits the last
# stage-2 tiles in two halves of K: 24 and 16 of them, ragged in N and T
SPLIT = [(2048, 6000, 2048, 1, 1500), (2048, 7000, 2048, 2, 900)]


@pytest.mark.parametrize("shape", SPLIT, ids=lambda s: "M{}N{}R{}l{}T{}".format(*s))
def test_fused_forward_split_tiles(dbf, shape):
    import ctypes
    M, N, R, ell, T = shape
    pairs = torch.cuda.get_device_properties(0).multi_processor_count // 2
    Lc = dbf.DbfLayerC(M, N, R, ell, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000)
    tiles = (ctypes.c_int32 * 3)()
    span = (ctypes.c_double * 2)()
    assert dbf._lib.dbf_debug_fused_schedule(ctypes.byref(Lc), T, pairs, tiles, span) == dbf.OK
    if pairs == 74:
        assert tiles[2] > 0
    rng = np.random.default_rng(sum(shape) + 12)
    # integer inputs with exact fp16 operands and fp32 sums: the two halves'
    # partial sums and their exchange are exact, so every element matches
    # the oracle bit for bit, and two calls agree
    L = exact_layer(rng, M, N, R, ell)
    x = rng.integers(-1, 2, size=(T, M)).astype(np.float32)
    a = run(dbf, L, x)
    assert np.array_equal(a, run(dbf, L, x))
    assert np.array_equal(a, oracle.forward(L, x))
    # random inputs, accumulating into y
    L = random_layer(rng, M, N, R, ell)
    x = S.to_bf16_bits(rng.standard_normal((T, M)))
    y_in = rng.standard_normal((T, N)).astype(np.float32)
    ref = oracle.forward(L, x, y_in=y_in, accumulate=True)
    assert rel_err(run(dbf, L, x, acc=True, y_in=y_in), ref) < TOL


@pytest.mark.parametrize("shape", [FUSED[2]], ids=lambda s: "M{}N{}R{}l{}T{}".format(*s))
def test_fused_forward_sign_flip_and_alpha_scaling(dbf, shape):
    # the two bit-exact invariants above, on the single-launch forward
    M, N, R, ell, T = shape
    rng = np.random.default_rng(64)
    L = random_layer(rng, M, N, R, ell)
    x = S.to_bf16_bits(rng.standard_normal((T, M)))
    y0 = run(dbf, L, x)
    flip = rng.random(R) < 0.5
    L.b1[:, flip] *= -1
    L.b2[flip, :] *= -1
    assert np.array_equal(run(dbf, L, x), y0)
    L.alpha[:] = S.to_f16_bits(2.0 * L.alpha.view(np.float16).astype(np.float64))
    assert np.array_equal(run(dbf, L, x), 2.0 * y0)
