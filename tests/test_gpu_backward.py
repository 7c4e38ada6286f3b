"""dbf_transpose_signs and dbf_backward on the GPU against the fp64 oracle.

Transposition is bit-exact. Gradients: max|g - g_ref| / max|g_ref| <= 2e-3
per output (the forward's bound; operands are fp16, accumulation fp32). At
the DBF MLP layer's full size (T = 2048, the bench's backward call) dx is
compared on sampled token rows (rows are independent) and the scale
gradients through Euler's identity, which holds at any size:
sum(alpha . dalpha) = sum(beta . dbeta) = sum(gamma . dgamma) =
sum(x . dx) = sum(dy . y).
"""
import numpy as np
import pytest
import torch

import dbf_synth as S
import oracle
from gpu_util import dev_layer, dev_x, random_layer, rel_err

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module")
def dbf():
    import double_binary_rank_b200 as m
    return m


@pytest.mark.parametrize("rows,k", [(1, 1), (33, 70), (256, 128), (130, 4100), (1000, 31)])
def test_transpose_bit_exact(dbf, rows, k):
    rng = np.random.default_rng(rows * 13 + k)
    s = rng.choice(np.array([-1, 1], dtype=np.int8), size=(rows, k))
    words = torch.from_numpy(oracle.pack(s).reshape(rows, -1).view(np.int32)).cuda()
    t = dbf.transpose_signs(words, rows, k)
    ref = oracle.pack(np.ascontiguousarray(s.T)).reshape(k, -1)
    assert np.array_equal(t.cpu().numpy().view(np.uint32), ref)
    back = dbf.transpose_signs(t, k, rows)
    assert torch.equal(back, words)


def gpu_grads(dbf, L, x, dy, **kw):
    dl = dev_layer(L)
    g = dbf.backward(dl, dev_x(x), dev_x(dy), **kw)
    torch.cuda.synchronize()
    return dl, g


CASES = [  # M, N, R, ell, T: several 128-row tiles, ragged token counts, ell*T across 256-column tiles
    (256, 384, 128, 1, 1), (256, 384, 128, 2, 37), (384, 256, 256, 1, 300), (128, 640, 384, 3, 100),
    (512, 128, 128, 2, 257),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "M{}N{}R{}l{}T{}".format(*c))
@pytest.mark.parametrize("kind", ["bf16", "f32"])
def test_backward_matches_oracle(dbf, case, kind):
    M, N, R, ell, T = case
    rng = np.random.default_rng(M + 3 * N + 7 * R + ell + T)
    L = random_layer(rng, M, N, R, ell)
    if kind == "bf16":
        x = S.to_bf16_bits(rng.standard_normal((T, M)))
        dy = S.to_bf16_bits(rng.standard_normal((T, N)))
    else:
        x = rng.standard_normal((T, M)).astype(np.float32)
        dy = rng.standard_normal((T, N)).astype(np.float32)
    ref = oracle.backward(L, x, dy)
    _, g = gpu_grads(dbf, L, x, dy)
    assert rel_err(g.dx.cpu().numpy(), ref.dx) < TOL
    assert rel_err(g.dalpha.cpu().numpy(), ref.dalpha) < TOL
    assert rel_err(g.dbeta.cpu().numpy(), ref.dbeta) < TOL
    assert rel_err(g.dgamma.cpu().numpy(), ref.dgamma) < TOL


# Shapes whose contractions are all at least 32 K steps deep: the sign GEMMs
# run as two launches (G4 with G3, G5 with G6) with tiles claimed at run
# time; two envelopes with ell T across 256-column tiles, ragged rows.
FUSED_CASES = [(2048, 2304, 2048, 2, 300), (2048, 2176, 2048, 1, 129)]


@pytest.mark.parametrize("case", FUSED_CASES, ids=lambda c: "M{}N{}R{}l{}T{}".format(*c))
def test_backward_claimed_tiles_match_oracle(dbf, case):
    M, N, R, ell, T = case
    rng = np.random.default_rng(M + 5 * N + ell + T)
    L = random_layer(rng, M, N, R, ell)
    x = S.to_bf16_bits(rng.standard_normal((T, M)))
    dy = S.to_bf16_bits(rng.standard_normal((T, N)))
    ref = oracle.backward(L, x, dy)
    dl, g = gpu_grads(dbf, L, x, dy)
    assert rel_err(g.dx.cpu().numpy(), ref.dx) < TOL
    assert rel_err(g.dalpha.cpu().numpy(), ref.dalpha) < TOL
    assert rel_err(g.dbeta.cpu().numpy(), ref.dbeta) < TOL
    assert rel_err(g.dgamma.cpu().numpy(), ref.dgamma) < TOL
    # without dalpha the second launch holds G6's tiles only
    only = dbf.backward(dl, dev_x(x), dev_x(dy), want=("dx", "dbeta"))
    torch.cuda.synchronize()
    assert only.dalpha is None
    assert rel_err(only.dx.cpu().numpy(), ref.dx) < TOL
    assert rel_err(only.dbeta.cpu().numpy(), ref.dbeta) < TOL


def test_backward_accumulate_and_optional_outputs(dbf):
    rng = np.random.default_rng(91)
    L = random_layer(rng, 256, 256, 128, 2)
    x = S.to_bf16_bits(rng.standard_normal((50, 256)))
    dy = S.to_bf16_bits(rng.standard_normal((50, 256)))
    ref = oracle.backward(L, x, dy)
    dl = dev_layer(L)
    xd, dyd = dev_x(x), dev_x(dy)
    base = dbf.Grads(torch.full((50, 256), 0.5, device="cuda"), torch.full((2, 256), -1.0, device="cuda"),
                     torch.full((2, 128), 2.0, device="cuda"), torch.full((2, 256), 0.25, device="cuda"))
    g = dbf.backward(dl, xd, dyd, grads=base, accumulate=True)
    torch.cuda.synchronize()
    assert rel_err(g.dx.cpu().numpy() - 0.5, ref.dx) < TOL
    assert rel_err(g.dalpha.cpu().numpy() + 1.0, ref.dalpha) < TOL
    assert rel_err(g.dbeta.cpu().numpy() - 2.0, ref.dbeta) < TOL
    assert rel_err(g.dgamma.cpu().numpy() - 0.25, ref.dgamma) < TOL
    only = dbf.backward(dl, xd, dyd, want=("dbeta",))
    torch.cuda.synchronize()
    assert only.dx is None and only.dalpha is None and only.dgamma is None
    assert rel_err(only.dbeta.cpu().numpy(), ref.dbeta) < TOL


def test_backward_rejects_unsupported_shape(dbf):
    rng = np.random.default_rng(92)
    L = random_layer(rng, 200, 256, 128, 1)
    dl = dev_layer(L)
    x = dev_x(S.to_bf16_bits(rng.standard_normal((4, 200))))
    dy = dev_x(S.to_bf16_bits(rng.standard_normal((4, 256))))
    with pytest.raises(dbf.DbfError) as e:
        dbf.backward(dl, x, dy, ws=torch.zeros(1 << 20, dtype=torch.uint8, device="cuda"))
    assert e.value.status == dbf.ERR_UNSUPPORTED


def test_dbf_mlp_full_size(dbf):
    w = S.WORKLOADS["dbf_mlp"]
    L = S.workload_layers(w)[0]
    T = 2048
    x = S.make_x(w.seed + 100, T, w.M, "bf16")
    dy = S.make_x(w.seed + 200, T, w.N, "bf16")
    dl, g = gpu_grads(dbf, L, x, dy)
    rows = S.sample_rows(w.seed, T, 16)
    ref = oracle.backward(L, x[rows], dy[rows])
    assert rel_err(g.dx.cpu().numpy()[rows], ref.dx) < TOL
    # Euler's identity over the whole batch
    y = oracle.forward(L, x)
    loss = float((y * S.bf16_bits_to_f32(dy).astype(np.float64)).sum())
    dec = lambda b: np.asarray(b, dtype=np.uint16).view(np.float16).astype(np.float64)
    sums = [
        float((dec(L.alpha) * g.dalpha.double().cpu().numpy()).sum()),
        float((dec(L.beta) * g.dbeta.double().cpu().numpy()).sum()),
        float((dec(L.gamma) * g.dgamma.double().cpu().numpy()).sum()),
        float((S.bf16_bits_to_f32(x).astype(np.float64) * g.dx.double().cpu().numpy()).sum()),
    ]
    scale = float(np.abs(y).max()) * np.sqrt(T * w.N)   # size of the terms of the sum
    for v in sums:
        assert abs(v - loss) <= TOL * scale, (v, loss)


def test_dbf_mlp_shape_elementwise(dbf):
    # The DBF MLP layer's full shape (4096 -> 11008, R = 5888) at 64 tokens:
    # every element of dx, dalpha, dbeta and dgamma against the oracle.
    w = S.WORKLOADS["dbf_mlp"]
    L = S.workload_layers(w)[0]
    T = 64
    x = S.make_x(w.seed + 300, T, w.M, "bf16")
    dy = S.make_x(w.seed + 400, T, w.N, "bf16")
    _, g = gpu_grads(dbf, L, x, dy)
    ref = oracle.backward(L, x, dy)
    assert rel_err(g.dx.cpu().numpy(), ref.dx) < TOL
    assert rel_err(g.dalpha.cpu().numpy(), ref.dalpha) < TOL
    assert rel_err(g.dbeta.cpu().numpy(), ref.dbeta) < TOL
    assert rel_err(g.dgamma.cpu().numpy(), ref.dgamma) < TOL


@pytest.mark.parametrize("case", [(256, 384, 128, 1, 37), (128, 256, 256, 2, 300), (384, 128, 128, 3, 5)],
                         ids=lambda c: "M{}N{}R{}l{}T{}".format(*c))
def test_sign_matrix_gradients(dbf, case):
    M, N, R, ell, T = case
    rng = np.random.default_rng(500 + M + N + R + ell + T)
    L = random_layer(rng, M, N, R, ell)
    x = S.to_bf16_bits(rng.standard_normal((T, M)))
    dy = S.to_bf16_bits(rng.standard_normal((T, N)))
    ref = oracle.backward(L, x, dy, want_signs=True)
    _, g = gpu_grads(dbf, L, x, dy, want=("dx", "dbeta", "db1", "db2"))
    assert g.dalpha is None and g.dgamma is None
    assert rel_err(g.db1.cpu().numpy(), ref.db1) < TOL
    assert rel_err(g.db2.cpu().numpy(), ref.db2) < TOL
    assert rel_err(g.dx.cpu().numpy(), ref.dx) < TOL
    # accumulate adds onto what is there
    dl = dev_layer(L)
    g2 = dbf.backward(dl, dev_x(x), dev_x(dy), grads=g, accumulate=True)
    torch.cuda.synchronize()
    assert rel_err(g2.db1.cpu().numpy(), 2 * ref.db1) < TOL
    assert rel_err(g2.db2.cpu().numpy(), 2 * ref.db2) < TOL


@pytest.mark.parametrize("tau", [0.0, 0.5, 2.0])
@pytest.mark.parametrize("hdt", [torch.float32, torch.bfloat16, torch.float16])
def test_ste_backward(dbf, tau, hdt):
    rng = np.random.default_rng(int(tau * 10) + 3)
    h = torch.from_numpy(rng.standard_normal((37, 129)).astype(np.float32) * 1.5).to(hdt)
    db = torch.from_numpy(rng.standard_normal((37, 129)).astype(np.float32))
    ref = oracle.ste_backward(db.numpy(), h.float().numpy(), tau)
    got = dbf.ste_backward(db.cuda(), h.cuda(), tau)
    torch.cuda.synchronize()
    if tau > 0:
        np.testing.assert_allclose(got.cpu().numpy(), ref, rtol=2e-6, atol=2e-6)
    else:
        np.testing.assert_array_equal(got.cpu().numpy(), ref.astype(np.float32))
    acc = dbf.ste_backward(db.cuda(), h.cuda(), tau, dh=got.clone(), accumulate=True)
    torch.cuda.synchronize()
    np.testing.assert_allclose(acc.cpu().numpy(), 2 * got.cpu().numpy(), rtol=1e-6, atol=1e-7)
