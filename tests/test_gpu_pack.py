"""dbf_pack_signs / dbf_unpack_signs on the GPU: bit-exact against the
oracle's packer (written from the layout definition in include/dbf.h)."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbf():
    import double_binary_rank_b200 as m
    return m


# rows of 1..2188 packed words: several 64-word runs per row, ragged runs and
# a ragged last word
SHAPES = [(1, 1), (1, 31), (3, 32), (5, 33), (17, 100), (16, 5888), (64, 4096), (4096, 64),
          (256, 16), (37, 1000), (3, 4136), (2, 2100), (7, 70000)]


@pytest.mark.parametrize("shape", SHAPES)
def test_pack_int8_bitexact(dbf, shape):
    rng = np.random.default_rng(shape[0] * 7919 + shape[1])
    s = rng.choice(np.array([-1, 1], dtype=np.int8), size=shape)
    words = dbf.pack_signs(torch.from_numpy(s).cuda())
    got = words.cpu().numpy().view(np.uint32)
    assert np.array_equal(got, oracle.pack(s))
    back = dbf.unpack_signs(words, *shape).cpu().numpy()
    assert np.array_equal(back, s)


@pytest.mark.parametrize("cols", [77, 4136])
@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
def test_pack_latents_sign_convention(dbf, dtype, cols):
    rng = np.random.default_rng(5)
    h = rng.standard_normal((9, cols)).astype(np.float32)
    h[0, :6] = [0.0, -0.0, 1e-3, -1e-3, 5.0, -5.0]
    ht = torch.from_numpy(h).to(dtype)
    hq = ht.float().numpy()                    # the values the kernel sees
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = dbf.pack_signs(ht.cuda(), status=status).cpu().numpy().view(np.uint32)
    assert np.array_equal(got, oracle.pack(oracle.sign_of_latent(hq)))
    assert int(status.item()) == 0


def test_pack_nan_latent_sets_status(dbf):
    h = torch.ones(4, 40)
    h[2, 7] = float("nan")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dbf.pack_signs(h.cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == dbf.ERR_INVALID_ARG


def test_pack_large_matrix_bitexact(dbf):
    # the full B1 of the DBF MLP layer: 11008 x 5888
    import dbf_synth as S
    w = S.WORKLOADS["dbf_mlp"]
    L = S.make_layer(w.seed, w.M, w.N, w.R, w.ell, w.sigma)
    got = dbf.pack_signs(torch.from_numpy(L.b1).cuda()).cpu().numpy().view(np.uint32)
    assert np.array_equal(got, oracle.pack(L.b1))
