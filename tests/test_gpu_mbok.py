"""dbf_mbok_forward (multi-boolean-kernel layer) on the GPU against the fp64 oracle.

Tolerance as the forward: max|y - y_ref| / max|y_ref| <= 2e-3 for fp32
outputs, bf16 outputs within half a bf16 ulp of y_ref plus that bound. At a
4096 x 4096, K = 3 layer with 2048 tokens (the bench's MBOK call) on sampled
token rows.
"""
import numpy as np
import pytest
import torch

import dbf_synth as S
import oracle
from gpu_util import TOL, bf16_ok, dev_x, host_y, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbf():
    import double_binary_rank_b200 as m
    return m


def dev_mbok(dbf, L):
    f16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.float16)).cuda()
    return dbf.MbokLayer.from_signs(torch.from_numpy(L.w).cuda(), f16(L.s_in), f16(L.s_out))


CASES = [(256, 200, 2, 37), (128, 384, 3, 300), (512, 129, 1, 1), (384, 1000, 4, 260)]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "M{}N{}K{}T{}".format(*c))
@pytest.mark.parametrize("acc", [False, True])
def test_mbok_matches_oracle(dbf, case, acc):
    M, N, K, T = case
    L = S.make_mbok_layer(0xDBF00100 + M + N + K + T, M, N, K)
    rng = np.random.default_rng(M + N + K + T)
    x = S.to_bf16_bits(rng.standard_normal((T, M)))
    y_in = rng.standard_normal((T, N)).astype(np.float32)
    ref = oracle.mbok_forward(L, x) + (y_in.astype(np.float64) if acc else 0.0)
    y = torch.from_numpy(y_in).cuda() if acc else None
    got = host_y(dbf.mbok_forward(dev_mbok(dbf, L), dev_x(x), y=y, accumulate=acc, y_dtype=torch.float32))
    assert rel_err(got, ref) < TOL


def test_mbok_fp32_input_bf16_output(dbf):
    L = S.make_mbok_layer(0xDBF00200, 256, 320, 2)
    rng = np.random.default_rng(9)
    x = rng.standard_normal((50, 256)).astype(np.float32)
    ref = oracle.mbok_forward(L, x)
    got = host_y(dbf.mbok_forward(dev_mbok(dbf, L), dev_x(x), y_dtype=torch.bfloat16))
    ok, worst = bf16_ok(got, ref)
    assert ok, worst


def test_mbok_large_sampled_rows(dbf):
    L = S.make_mbok_layer(0xDBF00006, 4096, 4096, 3)
    T = 2048
    x = S.make_x(0xDBF00006, T, 4096, "bf16")
    got = host_y(dbf.mbok_forward(dev_mbok(dbf, L), dev_x(x), y_dtype=torch.float32))
    rows = S.sample_rows(0xDBF00006, T, 24)
    ref = oracle.mbok_forward(L, x[rows])
    assert rel_err(got[rows], ref) < TOL
