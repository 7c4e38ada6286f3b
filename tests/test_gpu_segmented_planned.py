"""dbf_forward_segmented_planned (host segment tables, one forward per segment
on the path its length calls for) against the fp64 oracle's segmented forward.

Adapters of rank 128 (GEMM-eligible) and 32 (decode kernels only), segments
from 1 to 600 tokens, an adapter-less segment, accumulation; tolerance as the
forward (max|y - y_ref| / max|y_ref| <= 2e-3, fp32 output).
"""
import numpy as np
import pytest
import torch

import dbf_synth as S
import oracle
from gpu_util import TOL, dev_layer, dev_x, host_y, random_layer, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbf():
    import double_binary_rank_b200 as m
    return m


@pytest.mark.parametrize("acc", [False, True])
def test_planned_matches_oracle(dbf, acc):
    rng = np.random.default_rng(880 + int(acc))
    M = N = 512
    layers = [random_layer(rng, M, N, 128, 1), random_layer(rng, M, N, 32, 2), random_layer(rng, M, N, 256, 2)]
    lens = [600, 1, 37, 0, 300, 130, 5]
    ids = [0, 1, 2, 1, -1, 2, 0]
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(offs[-1])
    x = S.to_bf16_bits(rng.standard_normal((T, M)))
    y_in = rng.standard_normal((T, N)).astype(np.float32)
    ref = oracle.forward_segmented(layers, offs, ids, x, y_in=y_in if acc else None, accumulate=acc)
    dls = [dev_layer(L) for L in layers]
    y = torch.from_numpy(y_in).cuda() if acc else None
    got = host_y(dbf.forward_segmented_planned(dls, offs, ids, dev_x(x), y=y, accumulate=acc,
                                               y_dtype=torch.float32))
    assert rel_err(got, ref) < TOL


def test_planned_grouped_many_segments(dbf):
    # 60 segments of one GEMM-eligible shape (more than one grouped launch),
    # lengths from 1 to 300 tokens, two shape classes plus an ineligible one
    rng = np.random.default_rng(881)
    M, N = 256, 384
    layers = [random_layer(rng, M, N, 128, 1) for _ in range(5)] + [random_layer(rng, M, N, 256, 2),
                                                                     random_layer(rng, M, N, 64, 1)]
    lens = list(rng.integers(1, 40, size=57)) + [255, 256, 300]
    ids = [int(v) for v in rng.integers(0, 5, size=57)] + [5, 6, 5]
    ids[10] = -1
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(offs[-1])
    x = S.to_bf16_bits(rng.standard_normal((T, M)))
    ref = oracle.forward_segmented(layers, offs, ids, x)
    dls = [dev_layer(L) for L in layers]
    got = host_y(dbf.forward_segmented_planned(dls, offs, ids, dev_x(x), y_dtype=torch.float32))
    assert rel_err(got, ref) < TOL
