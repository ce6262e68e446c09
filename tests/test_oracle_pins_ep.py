"""Pins of the oracle's expert-parallel row placement (oracle_ep_plan).

The experts are split over `world` ranks in contiguous blocks; each rank owns
a contiguous chunk of the batch.  The receive layout at an owner (its experts
in order, inside an expert the copies of rank 0, 1, ..., each in token order)
must put every copy exactly where the single-GPU dispatch of the whole batch
puts it, shifted to the owner's first row: that ties the plan to the layer's
own dispatch (a separate oracle function, itself pinned by the hand-worked
example and brute force).
"""
import numpy as np
import pytest


def test_hand_worked_plan(orc):
    """world 2, E 4: counts [[1,2,3,4],[5,6,7,8]].  Owner 0 holds experts 0, 1:
    e0 = rank 0's 1 row then rank 1's 5 rows (rows 0..5), e1 from row 6
    (rank 0: 6..7, rank 1: 8..13), 14 rows; owner 1: e2 rows 0..9 (rank 1
    from 3), e3 from 10 (rank 1 from 14), 22 rows."""
    base, loff = orc.ep_plan(np.array([[1, 2, 3, 4], [5, 6, 7, 8]]))
    np.testing.assert_array_equal(base, [[0, 6, 0, 10], [1, 8, 3, 14]])
    np.testing.assert_array_equal(loff, [[0, 6, 14], [0, 10, 22]])


@pytest.mark.parametrize("world,E,K,T", [(2, 8, 2, 16), (4, 16, 4, 64), (8, 64, 8, 256),
                                         (8, 256, 8, 512), (1, 12, 3, 30), (3, 12, 4, 33)])
def test_plan_matches_the_single_gpu_dispatch(orc, world, E, K, T):
    rng = np.random.default_rng(world * 1000 + E + K)
    T -= T % world
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    Tr, El = T // world, E // world
    counts_all = np.stack([np.bincount(idx[r * Tr:(r + 1) * Tr].ravel(), minlength=E)
                           for r in range(world)]).astype(np.int32)
    base, loff = orc.ep_plan(counts_all)
    glob = orc.dispatch(idx, E, 1)
    for o in range(world):
        rows = int(loff[o, El])
        assert rows == counts_all[:, o * El:(o + 1) * El].sum()
        recv = np.full(rows, -1, np.int64)
        for r in range(world):
            seen = np.zeros(E, np.int64)
            for tl in range(Tr):
                t = r * Tr + tl
                for e in idx[t]:
                    if e // El != o:
                        continue
                    row = base[r, e] + seen[e]
                    seen[e] += 1
                    assert recv[row] == -1
                    recv[row] = t
        lo, hi = glob["offsets"][o * El], glob["offsets"][(o + 1) * El]
        np.testing.assert_array_equal(recv, glob["perm_token"][lo:hi])
        np.testing.assert_array_equal(loff[o, :El], glob["offsets"][o * El:(o + 1) * El] - lo)
