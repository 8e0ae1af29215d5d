"""The factorisation's block schedule, modelled in float64 on the CPU.

The GPU factor (reverse Cholesky H_d = R R^T, then U = R^-1) runs its block
columns from the last to the first, with the trailing updates and the sums
T_iq = sum_m R_im U_mq grouped over G block columns (see the schedule notes
in the factor source). This model replays the same schedule tile by tile in
program order, with the same ranges and K per product and with the planes of
U left undefined (NaN) wherever the GPU never writes them, and checks that
U^T U is H_d^-1 and U is upper triangular, for groups of 1 (step by step),
2, 3, 4 (the library's) and 8 block columns, ragged last blocks and final
groups of every length. A tile or range that the schedule forgets, updates
twice or reads too early breaks the identity or brings a NaN in.
"""

import numpy as np
import pytest

pytestmark = pytest.mark.filterwarnings("ignore")


def _schedule(K, t, last, G, group_from=16, seed=0, drop_far_tile=False):
    d = (K - 1) * t + last
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((3 * d, d))
    A0 = X.T @ X / d + 0.1 * np.eye(d)
    Aw = np.triu(A0).copy()                  # H_d, becoming R (upper part authoritative)
    U = np.zeros((d, d))                     # U, and the sums T in its unused upper part
    Upl = np.full((d, d), np.nan)            # the planes of U, written where U is formed
    Apl = np.zeros((d, t))                   # planes of the next column block above its diagonal
    cK = (K - 1) * t
    Apl[:cK, :last] = Aw[:cK, cK:cK + last]
    g = G if K >= group_from else 1
    blk = lambda b: slice(b * t, min(d, (b + 1) * t))
    cb = lambda b: min(d, b * t)
    Tpl = np.full((t, d), np.nan)           # planes of the next block row of T

    def first_of_group(k):
        return k + (K - 1 - k) % g

    def rows_ops(k):
        c0 = k * t
        k0 = first_of_group(k)
        LT = max(k0 - g + 1, 1)
        if k < K - 1:                        # block row k of U from T's block row k
            U[c0:c0 + t, c0 + t:] = -U[blk(k), blk(k)] @ Tpl[:t, c0 + t:]
            Upl[c0:c0 + t, c0 + t:] = U[c0:c0 + t, c0 + t:]
        if k > 0:
            if k > LT:                       # this step's term to the group's rows below it
                r0 = LT * t
                U[r0:c0, c0:] += Aw[r0:c0, c0:cb(k + 1)] @ Upl[c0:cb(k + 1), c0:]
            else:                            # all of the group's terms to the rows above it
                for q in range(k, k0):
                    kk = cb(q + 1) - c0
                    U[:c0, blk(q)] += Aw[:c0, c0:c0 + kk] @ Upl[c0:c0 + kk, blk(q)]
                kk = cb(k0 + 1) - c0
                U[:c0, cb(k0):] += Aw[:c0, c0:c0 + kk] @ Upl[c0:c0 + kk, cb(k0):]
            Tpl[:, c0:] = U[c0 - t:c0, c0:]

    def tile_upd(P, i, j):
        prod = P[blk(i)] @ P[blk(j)].T
        Aw[blk(i), blk(j)] -= np.triu(prod) if i == j else prod

    for k in range(K - 1, -1, -1):
        c0 = k * t
        bk = min(t, d - c0)
        # diag(k): D = R_kk R_kk^T (R_kk upper), U_kk = R_kk^-1
        D = np.triu(Aw[blk(k), blk(k)])
        D = D + np.triu(D, 1).T
        J = np.eye(bk)[::-1]
        Rkk = J @ np.linalg.cholesky(J @ D @ J) @ J
        U[blk(k), blk(k)] = np.linalg.inv(Rkk)
        Upl[blk(k), blk(k)] = np.triu(U[blk(k), blk(k)])
        if k == 0:
            rows_ops(k)
            break
        Ukk = U[blk(k), blk(k)]
        r0 = c0 - t
        # chain step(k): R_{k-1,k} and diagonal block k-1
        Rk1 = Apl[r0:c0, :bk] @ Ukk.T
        Aw[r0:c0, c0:c0 + bk] = Rk1
        Aw[r0:c0, r0:c0] -= np.triu(Rk1 @ Rk1.T)
        if k == 1:
            rows_ops(k)
            continue
        k0 = first_of_group(k)
        L = max(k0 - g + 1, 2)
        Aw[:r0, c0:c0 + bk] = Apl[:r0, :bk] @ Ukk.T          # panel rows < k-1
        if k > L:
            # own panel to the group's columns left of k (not tile (k-1, k-1))
            # and to diagonal tile (L-1, L-1); planes of column k-1
            P = Aw[:, c0:c0 + bk]
            tiles = [] if drop_far_tile else [(L - 1, L - 1)]
            tiles += [(i, j) for j in range(L, k) for i in range(j + 1) if (i, j) != (k - 1, k - 1)]
            for i, j in tiles:
                tile_upd(P, i, j)
        else:
            # all of the group's panels: column k-1 above its diagonal, then
            # every tile left of it
            P = Aw[:, c0:cb(k0 + 1)]
            for i in range(k - 1):
                tile_upd(P, i, k - 1)
            for j in range(k - 1):
                for i in range(j + 1):
                    tile_upd(P, i, j)
        for i in range(k - 1):
            Apl[blk(i), :t] = Aw[blk(i), blk(k - 1)]
        rows_ops(k)
    Ainv = np.linalg.inv(A0)
    return np.abs(U.T @ U - Ainv).max() / np.abs(Ainv).max(), np.abs(np.tril(U, -1)).max()


SHAPES = [(2, 4, 4), (7, 4, 1), (16, 4, 4), (17, 4, 3), (18, 4, 4), (19, 4, 2), (20, 4, 4), (21, 4, 1),
          (34, 4, 2)]


@pytest.mark.parametrize("G", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"K{s[0]}-last{s[2]}")
def test_grouped_factor_schedule_gives_the_exact_factor(shape, G):
    err, lower = _schedule(*shape, G=G)
    assert np.isfinite(err) and err < 1e-9, err
    assert lower == 0.0


def test_a_forgotten_tile_is_caught():
    """The check is not vacuous: leave the far diagonal tile (L-1, L-1) out
    of the early updates and the factor comes out wrong."""
    err, _ = _schedule(18, 4, 4, G=4, drop_far_tile=True)
    assert not err < 1e-6, err
