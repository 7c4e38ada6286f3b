"""Host-side schedule of the one-launch prefill forward (no GPU needed).

The library claims tiles at run time in order (stage-1 tiles, then stage-2
tiles, the last few split in two halves of K) and picks the number of split
tiles with a claim-order makespan model. These tests pin that model to
closed forms and invariants through dbf_debug_fused_schedule, which reads no
device memory.
"""
import ctypes
import math

import pytest


@pytest.fixture(scope="module")
def dbf():
    import double_binary_rank_b200 as m
    return m


def schedule(dbf, M, N, R, ell, T, pairs):
    L = dbf.DbfLayerC(M, N, R, ell, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000)
    tiles = (ctypes.c_int32 * 3)()
    span = (ctypes.c_double * 2)()
    st = dbf._lib.dbf_debug_fused_schedule(ctypes.byref(L), T, pairs, tiles, span)
    return st, list(tiles), list(span)


def test_tile_counts(dbf):
    # 256-row pair tiles of R (stage 1) and N (stage 2), 512-column blocks of
    # ell T (stage 1) and T (stage 2)
    st, tiles, _ = schedule(dbf, 4096, 11008, 5888, 1, 2048, 74)
    assert st == dbf.OK
    assert tiles[:2] == [23 * 4, 43 * 4]
    st, tiles, _ = schedule(dbf, 2048, 2500, 1024, 2, 1100, 74)
    assert st == dbf.OK
    assert tiles[:2] == [4 * math.ceil(2200 / 512), 10 * math.ceil(1100 / 512)]


def test_single_wave_closed_form(dbf):
    # every tile claimed at once (pairs >= tiles): the makespan is the longest
    # tile, K steps plus two; one stage-1 block, one stage-2 block
    M, N, R, T = 2048, 512, 2048, 1
    st, tiles, span = schedule(dbf, M, N, R, 1, T, 148)
    assert st == dbf.OK and tiles == [8, 2, 0]
    assert span[0] == max(M // 64, R // 64) + 2


def test_round_robin_closed_form(dbf):
    # equal K in both stages and a whole number of waves: the claim order
    # gives every pair the same number of tiles, makespan = waves * (K + 2)
    M = N = R = 8192
    st, tiles, span = schedule(dbf, M, N, R, 1, 8192, 64)
    assert st == dbf.OK
    n = tiles[0] + tiles[1]
    assert n % 64 == 0
    assert span[0] == (n // 64) * (8192 // 64 + 2)
    assert tiles[2] == 0   # nothing left to balance


def test_split_choice(dbf):
    # the DBF MLP layer at 2048 tokens: splitting the last stage-2 tiles in K
    # shortens the modelled makespan; the split count stays within its caps
    st, tiles, span = schedule(dbf, 4096, 11008, 5888, 1, 2048, 74)
    assert st == dbf.OK
    assert 0 < tiles[2] <= min(tiles[1], 64)
    assert span[1] < span[0]
    # more pairs than tiles: nothing to balance, no split
    st, tiles, span = schedule(dbf, 4096, 11008, 5888, 1, 256, 148)
    assert tiles[2] == 0 and span[1] == span[0]


@pytest.mark.parametrize("shape", [(4096, 11008, 5888, 1, 2048), (8192, 8192, 8192, 1, 8192),
                                   (2048, 2500, 1024, 2, 1100), (4096, 4096, 2048, 1, 1024)])
@pytest.mark.parametrize("pairs", [16, 74])
def test_split_never_worse_and_bounded(dbf, shape, pairs):
    st, tiles, span = schedule(dbf, *shape, pairs)
    assert st == dbf.OK
    assert span[1] <= span[0]
    # a lower bound: the total work spread evenly over the pairs
    M, N, R, ell, T = shape
    work = tiles[0] * (M // 64 + 2) + (tiles[1] - tiles[2]) * (ell * R // 64 + 2) + \
        tiles[2] * (ell * R // 64 + 6)
    assert span[1] >= work / pairs - 1e-9


def test_layers_outside_the_one_launch_forward(dbf):
    # a stage under 32 K steps, or M, R not multiples of 128
    assert schedule(dbf, 1024, 4096, 4096, 1, 2048, 74)[0] == dbf.ERR_UNSUPPORTED
    assert schedule(dbf, 2048, 4096, 1024, 1, 2048, 74)[0] == dbf.ERR_UNSUPPORTED
    assert schedule(dbf, 2100, 4096, 2048, 1, 2048, 74)[0] == dbf.ERR_UNSUPPORTED
    assert schedule(dbf, 2048, 4096, 2048, 1, 0, 74)[0] == dbf.ERR_INVALID_ARG
