"""dbf_svid (sign times the best rank-1 fit of |X|) and successive MBOK kernel
extraction on the GPU against the fp64 oracle.

Signs are bit-exact. The rank-1 factor comes from fp32 power iteration and
is stored in fp16, so the scale vectors are compared within 2e-3 of their
largest value; the residual update is checked elementwise against the same
stored scales; the extracted MBOK layer is checked through the library's
own MBOK forward against the dense matrix its signs and scales define.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbf():
    import double_binary_rank_b200 as m
    return m


def unpack_np(words, rows, k):
    return oracle.unpack(np.ascontiguousarray(words.cpu().numpy()).view(np.uint32).reshape(-1), rows, k)


# single-read kernel with 4, 8 and 12 float4 columns per thread (m % 4 == 0,
# m <= 12288, ragged last band); two-pass kernels for m % 4 != 0 and m > 12288
@pytest.mark.parametrize("n,m", [(300, 200), (1024, 4096), (77, 1000), (64, 5000), (40, 9000), (1, 12288),
                                 (129, 1001), (33, 12300)])
def test_svid_matches_oracle(dbf, n, m):
    rng = np.random.default_rng(n + m)
    X = rng.standard_normal((n, m)).astype(np.float32)
    X[0, :5] = 0.0          # sign(0) = +1
    S_ref, a_ref, b_ref = oracle.svid(X)
    Xd = torch.from_numpy(X).cuda()
    signs, a, b = dbf.svid(Xd, iters=30)
    torch.cuda.synchronize()
    assert np.array_equal(unpack_np(signs, n, m), S_ref)
    assert rel_err(a.float().cpu().numpy(), a_ref) < 2e-3
    assert rel_err(b.float().cpu().numpy(), b_ref) < 2e-3
    assert torch.equal(Xd.cpu(), torch.from_numpy(X))   # read only


def test_svid_stops_once_converged(dbf):
    # |X| exactly rank one: the second iterate is already the fixed point, so
    # the single-read path runs two iterations and passes it on; the result
    # is the oracle's
    rng = np.random.default_rng(5)
    n, m, iters = 512, 1024, 30
    a0 = rng.uniform(0.5, 2.0, n)
    b0 = rng.uniform(0.5, 2.0, m)
    X = (np.where(rng.random((n, m)) < 0.5, -1.0, 1.0) * np.outer(a0, b0)).astype(np.float32)
    S_ref, a_ref, b_ref = oracle.svid(X)
    scratch = dbf.alloc_workspace(int(dbf._lib.dbf_svid_scratch_bytes(n, m, iters)), torch.device("cuda", 0))
    signs, a, b = dbf.svid(torch.from_numpy(X).cuda(), iters=iters, scratch=scratch)
    torch.cuda.synchronize()
    assert dbf.svid_iterations(scratch, n, m, iters) <= 3
    assert np.array_equal(unpack_np(signs, n, m), S_ref)
    assert rel_err(a.float().cpu().numpy(), a_ref) < 2e-3
    assert rel_err(b.float().cpu().numpy(), b_ref) < 2e-3
    # a dense Gaussian matrix: stopping early gives the scales of a long run
    X = rng.standard_normal((300, 200)).astype(np.float32)
    Xd = torch.from_numpy(X).cuda()
    s30 = dbf.alloc_workspace(int(dbf._lib.dbf_svid_scratch_bytes(300, 200, 30)), torch.device("cuda", 0))
    _, a30, b30 = dbf.svid(Xd, iters=30, scratch=s30)
    _, a200, b200 = dbf.svid(Xd, iters=200)
    torch.cuda.synchronize()
    assert 1 <= dbf.svid_iterations(s30, 300, 200, 30) <= 30
    assert rel_err(a30.float().cpu().numpy(), a200.float().cpu().numpy()) < 1e-3
    assert rel_err(b30.float().cpu().numpy(), b200.float().cpu().numpy()) < 1e-3
    # the two-pass path (m % 4 != 0) runs every iteration
    X = rng.standard_normal((64, 1001)).astype(np.float32)
    s7 = dbf.alloc_workspace(int(dbf._lib.dbf_svid_scratch_bytes(64, 1001, 7)), torch.device("cuda", 0))
    dbf.svid(torch.from_numpy(X).cuda(), iters=7, scratch=s7)
    assert dbf.svid_iterations(s7, 64, 1001, 7) == 7


def test_svid_subtract_forms_the_residual(dbf):
    rng = np.random.default_rng(11)
    X = rng.standard_normal((256, 384)).astype(np.float32)
    Xd = torch.from_numpy(X.copy()).cuda()
    signs, a, b = dbf.svid(Xd, iters=30, subtract=True)
    torch.cuda.synchronize()
    a64 = a.float().double().cpu().numpy()
    b64 = b.float().double().cpu().numpy()
    expect = X.astype(np.float64) - np.where(X < 0, -1.0, 1.0) * np.outer(a64, b64)
    np.testing.assert_allclose(Xd.double().cpu().numpy(), expect, rtol=1e-6, atol=1e-5)


def test_mbok_extraction(dbf):
    rng = np.random.default_rng(12)
    N, M, K = 384, 512, 3
    W = rng.standard_normal((N, M)).astype(np.float32)
    layer = dbf.MbokLayer.extract(torch.from_numpy(W).cuda(), K, iters=30)
    torch.cuda.synchronize()
    # the first kernel's signs are sign(W)
    words = layer.w.cpu().numpy().view(np.uint32).reshape(N, -1)
    all_signs = oracle.unpack(np.ascontiguousarray(words).reshape(-1), N, K * M).reshape(N, K, M)
    assert np.array_equal(all_signs[:, 0, :], np.where(W < 0, -1, 1))
    so = layer.s_out.float().double().cpu().numpy()
    si = layer.s_in.float().double().cpu().numpy()
    W_hat = sum(all_signs[:, k, :] * np.outer(so[k], si[k]) for k in range(K))
    # residual norms against the oracle's own extraction
    _, _, _, norms = oracle.mbok_extract(W, K)
    assert abs(np.linalg.norm(W - W_hat) - norms[-1]) <= 1e-2 * norms[0]
    assert np.linalg.norm(W - W_hat) < norms[0]
    # the library's MBOK forward with the extracted layer
    x = rng.standard_normal((40, M)).astype(np.float32)
    y = dbf.mbok_forward(layer, torch.from_numpy(x).cuda(), y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert rel_err(y.double().cpu().numpy(), x.astype(np.float64) @ W_hat.T) < 2e-3
