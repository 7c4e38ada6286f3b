"""dbf_factorize (DBF page, section 2: alternating ADMM with the SVID
projection) on the GPU against the fp64 oracle.

The GPU runs the same steps in fp32 with an fp32 power-iteration SVID. An
fp32 re-run of the oracle's steps stays within ~1e-7 of fp64 on these cases,
so the bounds below (objective 1e-4 of |W|, fp16 scales 1e-3 of their
largest value, at most 0.1 % of the signs differing) leave room for the
blocked inverse and the power iteration while still catching a wrong step.
Cases: exact fixed points, the k = 1 Eckart-Young limit, the oracle's
trajectory from the same start (k a multiple of 4 and not, several 128-wide
GEMM tiles), and the DBF MLP weight size with properties that hold at any
size.
"""
import numpy as np
import pytest
import torch

import dbf_synth as S
import oracle
from gpu_util import dev_x, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbf():
    import double_binary_rank_b200 as m
    return m


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def unpack(words, rows, k):
    return oracle.unpack(np.ascontiguousarray(words.cpu().numpy()).view(np.uint32).reshape(-1), rows, k)


def f16(t):
    return t.float().double().cpu().numpy().reshape(-1)


def member(rng, r, c):
    Sg = rng.choice([-1.0, 1.0], size=(r, c))
    return np.exp(0.3 * rng.standard_normal(r))[:, None] * Sg * np.exp(0.3 * rng.standard_normal(c))[None, :]


@pytest.mark.parametrize("n,m,k", [(40, 30, 8), (130, 70, 33), (300, 260, 140)])
def test_exact_product_is_a_fixed_point(dbf, n, m, k):
    rng = np.random.default_rng(n * 7 + m + k)
    Ut, Vt = member(rng, n, k).astype(np.float32), member(rng, k, m).astype(np.float32)
    W = (Ut.astype(np.float64) @ Vt.astype(np.float64)).astype(np.float32)
    layer, obj = dbf.factorize(dev(W), dev(Ut), dev(Vt), outer=2, admm_iters=2, svid_iters=30)
    torch.cuda.synchronize()
    assert np.all(obj.cpu().numpy() <= 1e-4 * np.linalg.norm(W))
    assert np.array_equal(unpack(layer.b1, n, k), np.sign(Ut).astype(np.int8))
    assert np.array_equal(unpack(layer.b2, k, m), np.sign(Vt).astype(np.int8))
    What = (f16(layer.alpha)[:, None] * np.sign(Ut)) @ (f16(layer.beta)[:, None] * np.sign(Vt)) * f16(layer.gamma)
    assert rel_err(What, W.astype(np.float64)) < 2e-3   # fp16 scales


def test_rank_one_reaches_eckart_young(dbf):
    rng = np.random.default_rng(3)
    n, m = 200, 150
    W = (4.0 * np.outer(rng.standard_normal(n), rng.standard_normal(m)) + rng.standard_normal((n, m))).astype(np.float32)
    U0, V0 = rng.standard_normal((n, 1)), rng.standard_normal((1, m))
    _, obj = dbf.factorize(dev(W), dev(U0), dev(V0), outer=60, admm_iters=3, svid_iters=4)
    torch.cuda.synchronize()
    s = np.linalg.svd(W.astype(np.float64), compute_uv=False)
    best = np.sqrt(np.sum(s[1:] ** 2))
    o = obj.cpu().numpy()
    assert o[0] > 1.01 * best
    assert abs(float(o[-1]) - best) <= 1e-4 * np.linalg.norm(W)


@pytest.mark.parametrize("n,m,k,outer,admm", [(96, 80, 40, 2, 2), (130, 70, 33, 2, 3), (256, 192, 128, 3, 4),
                                              (300, 140, 200, 1, 2)])
def test_matches_oracle_from_the_same_start(dbf, n, m, k, outer, admm):
    W = S.make_weight(100 + n, n, m)
    U0, V0 = oracle.svd_init(W, min(k, min(n, m)))
    if k > U0.shape[1]:   # k above the rank: pad the start with a seeded random part
        Ur, Vr = S.make_factor_start(200 + n, n, m, k, scale=0.1)
        U0 = np.concatenate([U0, Ur[:, U0.shape[1]:]], axis=1)
        V0 = np.concatenate([V0, Vr[V0.shape[0]:]], axis=0)
    U0, V0 = U0.astype(np.float32), V0.astype(np.float32)
    ref = oracle.factorize(W, U0, V0, outer=outer, admm_iters=admm)
    layer, obj = dbf.factorize(dev(W), dev(U0), dev(V0), outer=outer, admm_iters=admm, svid_iters=40)
    torch.cuda.synchronize()
    nW = float(np.linalg.norm(W))
    assert np.abs(obj.cpu().numpy() - np.array(ref.objective)).max() <= 1e-4 * nW
    assert np.mean(unpack(layer.b1, n, k) != ref.A) <= 1e-3
    assert np.mean(unpack(layer.b2, k, m) != ref.B) <= 1e-3
    dec = lambda b: b.astype(np.uint16).view(np.float16).astype(np.float64)
    assert rel_err(f16(layer.alpha), dec(ref.alpha)) < 1e-3
    assert rel_err(f16(layer.beta), dec(ref.beta)) < 1e-3
    assert rel_err(f16(layer.gamma), dec(ref.gamma)) < 1e-3


def test_zero_outer_iterations_return_the_projected_start(dbf):
    W = S.make_weight(7, 64, 48)
    U0, V0 = S.make_factor_start(8, 64, 48, 20)
    ref = oracle.factorize(W, U0, V0, outer=0, admm_iters=1)
    layer, obj = dbf.factorize(dev(W), dev(U0), dev(V0), outer=0, svid_iters=40)
    torch.cuda.synchronize()
    assert np.array_equal(unpack(layer.b1, 64, 20), ref.A) and np.array_equal(unpack(layer.b2, 20, 48), ref.B)
    assert abs(float(obj[0]) - ref.objective[0]) <= 1e-4 * np.linalg.norm(W)


def test_dbf_mlp_weight_full_size(dbf):
    # 11008 x 4096 weight at k = 5888 (the DBF MLP layer's shape), one outer
    # iteration from a seeded random start
    w = S.WORKLOADS["dbf_mlp"]
    n, m, k = w.N, w.M, w.R
    W = S.make_weight(w.seed, n, m)
    U0, V0 = S.make_factor_start(w.seed + 1, n, m, k, scale=float(np.sqrt(np.mean(W.astype(np.float64) ** 2))))
    layer, obj = dbf.factorize(dev(W), dev(U0), dev(V0), outer=1, admm_iters=2, svid_iters=24)
    torch.cuda.synchronize()
    o = obj.cpu().numpy()
    assert np.all(np.isfinite(o)) and o[1] < o[0]
    # the returned layer through the library's forward against the oracle's
    L = S.Layer(M=m, N=n, R=k, ell=1, b1=unpack(layer.b1, n, k), b2=unpack(layer.b2, k, m),
                alpha=layer.alpha.cpu().numpy().view(np.uint16), beta=layer.beta.cpu().numpy().view(np.uint16),
                gamma=layer.gamma.cpu().numpy().view(np.uint16))
    x = S.make_x(w.seed + 5, 4, m, "bf16")
    y = dbf.forward(layer, dev_x(x), y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert rel_err(y.double().cpu().numpy(), oracle.forward(L, x)) < 2e-3
    # the approximation error the objective reports, on sampled rows
    rows = S.sample_rows(w.seed, n, 8)
    Bf = L.b2.astype(np.float64) * f16(layer.gamma)[None, :]
    What = (f16(layer.alpha)[rows, None] * L.b1[rows].astype(np.float64) * f16(layer.beta)[None, :]) @ Bf
    err_rows = np.linalg.norm(W[rows].astype(np.float64) - What, axis=1)
    assert np.all(err_rows < np.linalg.norm(W[rows].astype(np.float64), axis=1))
