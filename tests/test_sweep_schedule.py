"""The factorisation's blocked sweep inverse as the GPU schedules it, modelled
on the CPU (no GPU needed).

The library keeps the swept Gram matrix symmetric and maintains only its
lower triangle: the Gram product and every rank-bs trailing update compute
only the tiles (XM rows x BN columns, BN = 2 XM) that reach the lower
triangle, the panel of a pivot block is gathered from the block column below
the diagonal and the block row left of it, the fixup writes those two and
the pivot block, and the next pivot block is formed from E and P ahead of
the trailing update (lookahead); a mirror pass fills the upper triangle at
the end. This model follows those steps with the entries that no tile
computes poisoned (NaN), so a step that read one would spoil the result:
the result must equal -(G)^-1 and hold no NaN. It pins the schedule's
reading of the sweep (which entries are read and written, the order of the
lookahead), not the kernels' arithmetic, which the GPU parity tests check.
"""
import numpy as np
import pytest


def lower_tiles(k, xm, bn):
    """(row range, column range) of the tiles that reach the lower triangle."""
    tiles = []
    for c0 in range(0, k, bn):
        for r0 in range(0, k, xm):
            if r0 + xm > c0:   # some row of the tile is at or below some column
                tiles.append((slice(r0, min(r0 + xm, k)), slice(c0, min(c0 + bn, k))))
    return tiles


def lower_product(C, update, k, xm, bn):
    """C <- C + update on the lower tiles only (update computed from whole rows
    and columns, as each tile's K loop does)."""
    for rs, cs in lower_tiles(k, xm, bn):
        C[rs, cs] = C[rs, cs] + update[rs, cs]


def sweep_model(G, bsz, xm, bn):
    k = G.shape[0]
    A = np.full((k, k), np.nan)    # entries no tile of the lower-mode Gram product writes
    for rs, cs in lower_tiles(k, xm, bn):
        A[rs, cs] = G[rs, cs]
    blocks = [(p, min(bsz, k - p)) for p in range(0, k, bsz)]

    def panel(p0, bs):
        P = np.empty((k, bs))
        P[p0:] = A[p0:, p0:p0 + bs]          # block column at and below the diagonal
        P[:p0] = A[p0:p0 + bs, :p0].T        # block row left of it
        return P

    P = panel(*blocks[0])
    D = np.linalg.inv(P[0:blocks[0][1]])   # the pivot block's inverse
    for j, (p0, bs) in enumerate(blocks):
        E = P @ D
        nxt = blocks[j + 1] if j + 1 < len(blocks) else None
        if nxt is not None:
            p1, bn1 = nxt
            # the next pivot block as the update will leave it, formed first
            T = A[p1:p1 + bn1, p1:p1 + bn1] - E[p1:p1 + bn1] @ P[p1:p1 + bn1].T
            assert not np.isnan(T).any()
            D_next = np.linalg.inv(T)
        lower_product(A, -(E @ P.T), k, xm, bn)
        # fixup: the pivot block, the block column below it, the block row left of it
        A[p0:p0 + bs, p0:p0 + bs] = -D
        A[p0 + bs:, p0:p0 + bs] = E[p0 + bs:]
        A[p0:p0 + bs, :p0] = E[:p0].T
        if nxt is not None:
            P = panel(*nxt)
            D = D_next
    # mirror: the upper triangle from the lower
    iu = np.triu_indices(k, 1)
    A[iu] = A.T[iu]
    return A


@pytest.mark.parametrize("k,bsz", [(40, 8), (37, 8), (64, 16), (8, 8), (9, 8), (100, 12)])
def test_sweep_schedule_inverts_and_reads_only_maintained_entries(k, bsz):
    rng = np.random.default_rng(k * 100 + bsz)
    V = rng.standard_normal((k, 3 * k))
    G = V @ V.T + np.trace(V @ V.T) / k * np.eye(k)   # Gram + rho I, rho = trace / k
    A = sweep_model(G, bsz, xm=bsz, bn=2 * bsz)
    assert not np.isnan(A).any()
    np.testing.assert_allclose(A, -np.linalg.inv(G), rtol=1e-9, atol=1e-12 * np.abs(np.linalg.inv(G)).max())


def test_lower_tiles_cover_the_lower_triangle_once():
    # every entry on or below the diagonal lies in exactly one lower tile;
    # the tiles of column block c start at row tile 2c (BN = 2 XM)
    k, xm, bn = 50, 8, 16
    count = np.zeros((k, k), dtype=int)
    for rs, cs in lower_tiles(k, xm, bn):
        count[rs, cs] += 1
        assert rs.start >= 2 * (cs.start // bn) * xm
    il = np.tril_indices(k)
    assert (count[il] == 1).all()
    assert count.max() == 1
