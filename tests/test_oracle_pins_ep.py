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


def test_hand_worked_token_plan(orc):
    """world 2, E 4 (owner 0: experts 0, 1; owner 1: 2, 3), K 2.  Rank 0's
    tokens: t0 -> {0, 1} (owner 0 only), t1 -> {1, 2} (both owners); rank 1's:
    t2 -> {2, 3} (owner 1), t3 -> {0, 3} (both).  Owner 0 receives rank 0's
    t0, t1 (rows 0, 1) then rank 1's t3 (row 2); owner 1 receives rank 0's t1
    (row 0), then rank 1's t2, t3 (rows 1, 2)."""
    slot0, cnt0 = orc.ep_token_plan(np.array([[0, 1], [1, 2]]), 4, 2)
    slot1, cnt1 = orc.ep_token_plan(np.array([[2, 3], [0, 3]]), 4, 2)
    np.testing.assert_array_equal(slot0, [[0, -1], [1, 0]])
    np.testing.assert_array_equal(cnt0, [2, 1])
    np.testing.assert_array_equal(slot1, [[-1, 0], [0, 1]])
    np.testing.assert_array_equal(cnt1, [1, 2])
    np.testing.assert_array_equal(orc.ep_token_base(np.stack([cnt0, cnt1])), [[0, 0], [2, 1]])


@pytest.mark.parametrize("world,E,G,K,M,T", [(2, 8, 2, 2, 1, 16), (4, 16, 4, 4, 2, 64),
                                             (8, 64, 8, 8, 4, 256), (8, 256, 8, 8, 4, 512),
                                             (4, 32, 8, 8, 4, 96), (1, 12, 3, 3, 3, 30)])
def test_token_plan_fans_out_to_the_single_gpu_dispatch(orc, world, E, G, K, M, T):
    """Each token crosses once to each owner holding one of its experts; the
    owner's fan-out of those rows, indexed through the copy rows of the expert
    plan, must reproduce the single-GPU dispatch's perm_token for its experts,
    and with owners = groups the per-owner token counts are the dispatch's
    send_tok (both from a separate, pinned oracle function).  Routings are
    node-limited: M of G groups, K/M experts in each."""
    rng = np.random.default_rng(world * 7919 + E + K)
    gsz, kpg = E // G, K // M
    idx = np.stack([np.concatenate([g * gsz + rng.permutation(gsz)[:kpg]
                                    for g in rng.permutation(G)[:M]]) for _ in range(T)])
    idx = idx.astype(np.int32)
    Tr, El = T // world, E // world
    plans = [orc.ep_token_plan(idx[r * Tr:(r + 1) * Tr], E, world) for r in range(world)]
    tok_counts_all = np.stack([p[1] for p in plans])
    tok_base = orc.ep_token_base(tok_counts_all)
    counts_all = np.stack([np.bincount(idx[r * Tr:(r + 1) * Tr].ravel(), minlength=E)
                           for r in range(world)]).astype(np.int32)
    base, loff = orc.ep_plan(counts_all)
    glob = orc.dispatch(idx, E, G)
    if world == G:
        np.testing.assert_array_equal(tok_counts_all, glob["send_tok"])
    for o in range(world):
        n_tok = int(tok_counts_all[:, o].sum())
        recv_tok = np.full(n_tok, -1, np.int64)          # global token of each row
        rows = int(loff[o, El])
        fan = np.full(rows, -1, np.int64)                # copy row -> token row
        for r in range(world):
            slot = plans[r][0]
            seen = np.zeros(E, np.int64)
            for tl in range(Tr):
                t = r * Tr + tl
                if slot[tl, o] >= 0:
                    row = tok_base[r, o] + slot[tl, o]
                    assert recv_tok[row] == -1
                    recv_tok[row] = t
                else:
                    assert all(int(e) // El != o for e in idx[t])
                for e in idx[t]:
                    if e // El != o:
                        continue
                    crow = base[r, e] + seen[e]
                    seen[e] += 1
                    fan[crow] = tok_base[r, o] + slot[tl, o]
        assert (recv_tok >= 0).all() and (fan >= 0).all()
        lo, hi = glob["offsets"][o * El], glob["offsets"][(o + 1) * El]
        np.testing.assert_array_equal(recv_tok[fan], glob["perm_token"][lo:hi])


def _node_limited(rng, T, E, G, K, M):
    gsz, kpg = E // G, K // M
    return np.stack([np.concatenate([g * gsz + rng.permutation(gsz)[:kpg]
                                     for g in rng.permutation(G)[:M]])
                     for _ in range(T)]).astype(np.int32)


def _fanout_reproduces_dispatch(orc, idx, E, G, world, plans, tok_base, base, loff):
    """True when the owners' fan-out of the token rows, placed by (plans,
    tok_base) and indexed through the copy rows of (base, loff), reproduces
    the single-GPU dispatch's perm_token for every owner."""
    T = idx.shape[0]
    Tr, El = T // world, E // world
    glob = orc.dispatch(idx, E, G)
    for o in range(world):
        n_tok = int(sum(int(p[1][o]) for p in plans))
        recv_tok = np.full(n_tok, -1, np.int64)
        rows = int(loff[o, El])
        fan = np.full(rows, -1, np.int64)
        for r in range(world):
            slot = plans[r][0]
            seen = np.zeros(E, np.int64)
            for tl in range(Tr):
                t = r * Tr + tl
                mine = [int(e) for e in idx[t] if int(e) // El == o]
                if (slot[tl, o] >= 0) != bool(mine):
                    return False
                if not mine:
                    continue
                row = int(tok_base[r, o] + slot[tl, o])
                if not 0 <= row < n_tok or recv_tok[row] != -1:
                    return False
                recv_tok[row] = t
                for e in mine:
                    crow = int(base[r, e] + seen[e])
                    seen[e] += 1
                    if not 0 <= crow < rows:
                        return False
                    fan[crow] = row
        if (recv_tok < 0).any() or (fan < 0).any():
            return False
        lo, hi = glob["offsets"][o * El], glob["offsets"][(o + 1) * El]
        if not np.array_equal(recv_tok[fan], glob["perm_token"][lo:hi]):
            return False
    return True


def test_planted_mistakes_in_the_placements_are_caught(orc):
    """The fan-out property accepts the oracle's placements and rejects each
    of these planted mistakes: ranks swapped in the copy placement, a token
    slot off by one, a token counted at an owner it has no expert at, the
    token bases taken from the wrong rank."""
    world, E, G, K, M, T = 4, 16, 4, 4, 2, 64
    idx = _node_limited(np.random.default_rng(3), T, E, G, K, M)
    Tr = T // world
    plans = [orc.ep_token_plan(idx[r * Tr:(r + 1) * Tr], E, world) for r in range(world)]
    tok_base = orc.ep_token_base(np.stack([p[1] for p in plans]))
    counts_all = np.stack([np.bincount(idx[r * Tr:(r + 1) * Tr].ravel(), minlength=E)
                           for r in range(world)]).astype(np.int32)
    base, loff = orc.ep_plan(counts_all)
    assert _fanout_reproduces_dispatch(orc, idx, E, G, world, plans, tok_base, base, loff)
    # ranks 0 and 1 swapped in the copy placement
    swapped = base.copy()
    swapped[[0, 1]] = swapped[[1, 0]]
    assert not _fanout_reproduces_dispatch(orc, idx, E, G, world, plans, tok_base, swapped, loff)
    # one token's slot at an owner off by one
    slot0 = plans[0][0].copy()
    o = int(idx[0][0]) // (E // world)
    slot0[0, o] += 1
    bad = [(slot0, plans[0][1])] + plans[1:]
    assert not _fanout_reproduces_dispatch(orc, idx, E, G, world, bad, tok_base, base, loff)
    # a token sent to an owner holding none of its experts
    slot0 = plans[0][0].copy()
    t_none, o_none = next((t, o) for t in range(Tr) for o in range(world) if slot0[t, o] < 0)
    slot0[t_none, o_none] = 0
    bad = [(slot0, plans[0][1])] + plans[1:]
    assert not _fanout_reproduces_dispatch(orc, idx, E, G, world, bad, tok_base, base, loff)
    # token bases of rank 1 used for rank 2
    tb = tok_base.copy()
    tb[2] = tb[1]
    assert not _fanout_reproduces_dispatch(orc, idx, E, G, world, plans, tb, base, loff)


try:
    from hypothesis import given, settings, strategies as st
except ImportError:  # pragma: no cover - hypothesis ships with the test environment
    given = None

if given is not None:
    @st.composite
    def _ep_case(draw):
        world = draw(st.sampled_from([1, 2, 3, 4]))
        groups_per_rank = draw(st.integers(1, 2))
        G = world * groups_per_rank
        gsz = draw(st.integers(1, 4))
        E = G * gsz
        M = draw(st.integers(1, G))
        kpg = draw(st.integers(1, gsz))
        Tr = G * draw(st.integers(1, 4))
        seed = draw(st.integers(0, 2**31 - 1))
        return world, E, G, M * kpg, M, Tr * world, seed

    @settings(max_examples=40, deadline=None)
    @given(_ep_case())
    def test_random_placements_fan_out_to_the_single_gpu_dispatch(orc, case):
        """Random node-limited routings, worlds and group layouts: the expert
        and token placements together reproduce the single-GPU dispatch."""
        world, E, G, K, M, T, seed = case
        idx = _node_limited(np.random.default_rng(seed), T, E, G, K, M)
        Tr = T // world
        plans = [orc.ep_token_plan(idx[r * Tr:(r + 1) * Tr], E, world) for r in range(world)]
        tok_base = orc.ep_token_base(np.stack([p[1] for p in plans]))
        counts_all = np.stack([np.bincount(idx[r * Tr:(r + 1) * Tr].ravel(), minlength=E)
                               for r in range(world)]).astype(np.int32)
        base, loff = orc.ep_plan(counts_all)
        assert _fanout_reproduces_dispatch(orc, idx, E, G, world, plans, tok_base, base, loff)
