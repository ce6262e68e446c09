"""Property-based pins of the oracle: random layer sizes and inputs drawn by
hypothesis, checked against brute force and against invariants that any
correct node-limited router and counting-sort dispatch must satisfy.

Selection: the chosen set is the brute-force optimum (largest sum of biased
affinities over every K-subset of the experts of every admissible set of M
groups, groups ranked by their top-(K/M) sums), K distinct experts within M
groups, descending order, gates summing to one.  Dispatch: a permutation whose
segments are sorted by expert then token, with counts, offsets and both send
matrices equal to direct counts.
"""
import itertools

import numpy as np
from hypothesis import given, settings, strategies as st


@st.composite
def layer(draw):
    G = draw(st.sampled_from([1, 2, 3, 4]))
    gsz = draw(st.integers(1, 5))
    E = G * gsz
    M = draw(st.integers(1, G))
    kpg = draw(st.integers(1, gsz))
    K = M * kpg
    T = G * draw(st.integers(1, 6))
    seed = draw(st.integers(0, 2**31 - 1))
    return E, G, K, M, T, seed


@settings(max_examples=60, deadline=None)
@given(layer())
def test_select_is_the_bruteforce_optimum(orc, case):
    E, G, K, M, T, seed = case
    rng = np.random.default_rng(seed)
    s = rng.uniform(0.01, 0.99, size=(T, E)).astype(np.float32)
    bias = rng.normal(0, 0.2, size=E).astype(np.float32)
    idx, w, gscore = orc.select(s, bias, G, K, M, want_group_score=True)
    gsz, kpg = E // G, K // M
    for t in range(T):
        b = (s[t] + bias).astype(np.float32).astype(np.float64)
        if len(set(b.tolist())) < E:
            continue  # exact ties: the tie rule has its own pins
        row = idx[t].tolist()
        assert len(set(row)) == K and all(0 <= e < E for e in row)
        groups = {e // gsz for e in row}
        assert len(groups) <= M
        assert all(b[row[j]] > b[row[j + 1]] for j in range(K - 1))
        # group scores: sum of each group's top-(K/M) biased affinities
        gs = [sorted(b[g * gsz:(g + 1) * gsz], reverse=True)[:kpg] for g in range(G)]
        np.testing.assert_allclose(gscore[t], [sum(v) for v in gs], rtol=1e-6, atol=1e-6)
        # the kept groups are the M best (scores distinct here with probability one)
        order = sorted(range(G), key=lambda g: (-sum(gs[g]), g))[:M]
        assert groups <= set(order)
        allowed = [e for e in range(E) if e // gsz in order]
        best = max(itertools.combinations(allowed, K), key=lambda c: sum(b[i] for i in c))
        assert set(row) == set(best)
        np.testing.assert_allclose(float(w[t].astype(np.float64).sum()), 1.0, rtol=0, atol=1e-6)
        assert (w[t] > 0).all()


@settings(max_examples=60, deadline=None)
@given(layer())
def test_dispatch_is_a_sorted_permutation(orc, case):
    E, G, K, M, T, seed = case
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    d = orc.dispatch(idx, E, G)
    n = T * K
    perm, inv = d["perm_token"], d["inv_perm"]
    # inv_perm is a bijection onto the rows, and perm_token undoes it
    assert sorted(inv.ravel().tolist()) == list(range(n))
    for t in range(T):
        for j in range(K):
            assert perm[inv[t, j]] == t
    # rows are sorted by (expert, token); counts and offsets are direct counts
    expert_of_row = np.empty(n, np.int64)
    for t in range(T):
        for j in range(K):
            expert_of_row[inv[t, j]] = idx[t, j]
    keys = list(zip(expert_of_row.tolist(), perm.tolist()))
    assert keys == sorted(keys)
    np.testing.assert_array_equal(d["counts"], np.bincount(idx.ravel(), minlength=E))
    np.testing.assert_array_equal(d["offsets"], np.concatenate([[0], np.cumsum(d["counts"])]))
    # send matrices: copies and (token, destination group) pairs per source group
    gsz, chunk = E // G, T // G
    send = np.zeros((G, G), np.int64)
    send_tok = np.zeros((G, G), np.int64)
    for t in range(T):
        dst = [int(e) // gsz for e in idx[t]]
        for g in dst:
            send[t // chunk, g] += 1
        for g in set(dst):
            send_tok[t // chunk, g] += 1
    np.testing.assert_array_equal(d["send"], send)
    np.testing.assert_array_equal(d["send_tok"], send_tok)
