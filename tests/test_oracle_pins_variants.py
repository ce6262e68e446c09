"""Pins of the oracle's routing variants against facts outside the oracle.

* sqrt(softplus) affinity (the V4 form of "MoE + Expert-Parallel Overlap
  (Exp08)", Implemented): closed forms, asymptotes and numpy's logaddexp.
* Hash router (same passage; rule as read in the oracle's header): the
  published inverse of lowbias32, the routing invariants (K distinct experts,
  exactly M groups with K/M each, gates 1/K, keyed by token id only) and
  uniformity of the draws.
* Per-expert bias update (same passage; DeepSeek-V3's sign rule): hand-worked
  cases, exact integer mean comparison, fp32 add rounding.
"""
import numpy as np
import pytest
import torch

import synth


def _bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _bf16_np(t):
    return t.float().numpy().astype(np.float64)


def _sqrt_softplus(L):
    return np.sqrt(np.logaddexp(0.0, np.asarray(L, dtype=np.float64)))


# ---------------------------------------------------------------- sqrt(softplus)
def test_sqrt_softplus_zero_logit_is_sqrt_ln2(orc):
    x = _bf16(np.random.default_rng(0).normal(size=(3, 32)))
    s = orc.router_scores(x, np.zeros((4, 32), np.float32), affinity=1)
    assert (s == np.float32(np.sqrt(np.log(2.0)))).all()


def test_sqrt_softplus_offsets_match_logaddexp_and_asymptotes(orc):
    """e = 0, so L = o exactly; both tails of softplus are exercised."""
    off = np.array([-80, -40, -5, -1e-3, 0, 1e-3, 3, 20, 50, 88], np.float32)
    x = _bf16(np.ones((2, 16)))
    s = orc.router_scores(x, np.zeros((off.size, 16), np.float32), off, affinity=1)
    want = _sqrt_softplus(off.astype(np.float64)).astype(np.float32)
    np.testing.assert_array_equal(s[0], want)
    # tails: softplus(L) ~ e^L for L << 0, ~ L for L >> 0
    np.testing.assert_allclose(s[0, 0], np.exp(-40.0), rtol=1e-6)
    np.testing.assert_allclose(s[0, -1], np.sqrt(88.0), rtol=1e-6)
    assert np.all(np.diff(s[0].astype(np.float64)) > 0)  # strictly increasing here


def test_sqrt_softplus_random_against_numpy(orc):
    rng = np.random.default_rng(3)
    x = _bf16(rng.normal(size=(40, 128)))
    e = rng.normal(0, 0.1, size=(24, 128)).astype(np.float32)
    off = rng.normal(0, 1, size=24).astype(np.float32)
    s = orc.router_scores(x, e, off, affinity=1)
    L = _bf16_np(x) @ e.astype(np.float64).T + off.astype(np.float64)
    np.testing.assert_allclose(s, _sqrt_softplus(L), rtol=1.2e-7, atol=0)


def test_sqrt_softplus_keeps_the_single_group_ranking(orc):
    """G = M = 1: selection is a pure ranking, and sqrt(softplus) is increasing
    like the sigmoid, so both affinities pick the same experts (zero bias)."""
    rng = np.random.default_rng(4)
    x = _bf16(rng.normal(size=(64, 64)))
    e = rng.normal(0, 0.2, size=(32, 64)).astype(np.float32)
    s0 = orc.router_scores(x, e, affinity=0)
    s1 = orc.router_scores(x, e, affinity=1)
    zero = np.zeros(32, np.float32)
    i0, _ = orc.select(s0, zero, 1, 6, 1)
    i1, w1 = orc.select(s1, zero, 1, 6, 1)
    np.testing.assert_array_equal(i0, i1)
    np.testing.assert_allclose(w1.sum(axis=1), 1.0, rtol=1e-6)


def test_layer_with_sqrt_softplus_equals_composed_steps(orc):
    shape = synth.MoeShape("v4mini", T=12, d=32, E=8, G=4, K=4, M=2, d_ff=16, n_shared=1,
                           d_ff_shared=8, x_sigma=1, e_sigma=1, bias_sigma=0.1)
    rng = np.random.default_rng(5)
    x = _bf16(rng.normal(size=(12, 32)))
    e = rng.normal(0, 0.3, size=(8, 32)).astype(np.float32)
    bias = rng.normal(0, 0.1, size=8).astype(np.float32)
    Wg = [_bf16(rng.normal(size=(16, 32)) / 6) for _ in range(8)]
    Wu = [_bf16(rng.normal(size=(16, 32)) / 6) for _ in range(8)]
    Wd = [_bf16(rng.normal(size=(32, 16)) / 4) for _ in range(8)]
    Sg, Su = _bf16(rng.normal(size=(1, 8, 32)) / 6), _bf16(rng.normal(size=(1, 8, 32)) / 6)
    Sd = _bf16(rng.normal(size=(1, 32, 8)) / 3)
    out, idx, w, sc = orc.layer_rows(range(12), shape, x, e, bias, Wg, Wu, Wd, Sg, Su, Sd,
                                     router=orc.ROUTER_SQRT_SOFTPLUS)
    np.testing.assert_array_equal(sc, orc.router_scores(x, e, affinity=1))
    i2, w2 = orc.select(sc, bias, 4, 4, 2)
    np.testing.assert_array_equal(idx, i2)
    np.testing.assert_array_equal(w, w2)
    want = np.stack([orc.shared_row(x[t], Sg, Su, Sd) + sum(
        float(w[t, j]) * orc.ffn_row(x[t], Wg[idx[t, j]], Wu[idx[t, j]], Wd[idx[t, j]])
        for j in range(4)) for t in range(12)])
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- hash router
def _lowbias32_inverse(x):
    """The published inverse of lowbias32 (hash-prospector): undoes it exactly."""
    m = 0xFFFFFFFF
    x ^= x >> 16
    x = (x * 0x43021123) & m
    x ^= (x >> 15) ^ (x >> 30)
    x = (x * 0x1D69E2A5) & m
    x ^= x >> 16
    return x


def test_lowbias32_is_undone_by_its_published_inverse(orc):
    assert orc.lowbias32(0) == 0
    vals = list(np.random.default_rng(6).integers(0, 2**32, size=300, dtype=np.uint64))
    vals += [1, 2, 0xFFFFFFFF, 0x80000000, 0xDEADBEEF]
    outs = set()
    for v in vals:
        h = orc.lowbias32(int(v))
        assert _lowbias32_inverse(h) == int(v)
        outs.add(h)
    assert len(outs) == len(set(int(v) for v in vals))


@pytest.mark.parametrize("E,G,K,M", [(8, 2, 2, 1), (16, 4, 4, 2), (64, 8, 8, 4), (256, 8, 8, 4),
                                     (12, 3, 6, 3), (32, 1, 5, 1), (9, 9, 9, 9)])
def test_hash_route_invariants(orc, E, G, K, M):
    ids = np.random.default_rng(7).integers(0, 2**40, size=500)
    idx, w = orc.hash_route(ids, E, G, K, M)
    gsz, kpg = E // G, K // M
    assert (w == np.float32(1.0 / K)).all()
    assert idx.min() >= 0 and idx.max() < E
    for t in range(len(ids)):
        row = idx[t]
        assert len(set(row.tolist())) == K
        groups = row // gsz
        for gi in range(M):  # slots in blocks of K/M, one group per block
            blk = groups[gi * kpg:(gi + 1) * kpg]
            assert (blk == blk[0]).all()
        assert len(set(groups.tolist())) == M


def test_hash_route_depends_on_the_token_id_only(orc):
    ids = np.array([5, 17, 5, 2**33 + 5, 17, 0], np.int64)
    idx, _ = orc.hash_route(ids, 64, 8, 8, 4)
    np.testing.assert_array_equal(idx[0], idx[2])
    np.testing.assert_array_equal(idx[1], idx[4])
    assert not np.array_equal(idx[0], idx[3])  # the high word of the id matters


def test_hash_route_full_selection_is_every_expert(orc):
    """K = E (so M = G): each token takes all experts, in some order."""
    idx, _ = orc.hash_route(np.arange(50), 12, 4, 12, 4)
    for row in idx:
        assert sorted(row.tolist()) == list(range(12))


def test_hash_route_is_uniform(orc):
    """Each expert, each first group and each within-group slot is drawn
    uniformly: chi-square far below a 1e-6 tail bound (catches an off-by-one
    in the shuffle that never picks the last candidate)."""
    from scipy.stats import chi2
    E, G, K, M, n = 32, 8, 4, 2, 40000
    idx, _ = orc.hash_route(np.arange(n), E, G, K, M)

    def stat(obs):
        exp = obs.sum() / obs.size
        return ((obs - exp) ** 2 / exp).sum(), obs.size - 1

    for obs in (np.bincount(idx.ravel(), minlength=E),       # expert load
                np.bincount(idx[:, 0] // (E // G), minlength=G),  # first group
                np.bincount(idx[:, 0] % (E // G), minlength=E // G),  # first pick in group
                np.bincount(idx[:, 1] % (E // G), minlength=E // G)):  # second pick
        s, dof = stat(obs.astype(np.float64))
        assert obs.min() > 0
        assert s < chi2.isf(1e-6, dof)


def test_layer_with_hash_router_equals_composed_steps(orc):
    shape = synth.MoeShape("hmini", T=10, d=32, E=8, G=4, K=4, M=2, d_ff=16, n_shared=1,
                           d_ff_shared=8, x_sigma=1, e_sigma=1, bias_sigma=0)
    rng = np.random.default_rng(8)
    x = _bf16(rng.normal(size=(10, 32)))
    Wg = [_bf16(rng.normal(size=(16, 32)) / 6) for _ in range(8)]
    Wu = [_bf16(rng.normal(size=(16, 32)) / 6) for _ in range(8)]
    Wd = [_bf16(rng.normal(size=(32, 16)) / 4) for _ in range(8)]
    Sg, Su = _bf16(rng.normal(size=(1, 8, 32)) / 6), _bf16(rng.normal(size=(1, 8, 32)) / 6)
    Sd = _bf16(rng.normal(size=(1, 32, 8)) / 3)
    tok = rng.integers(0, 1000, size=10)
    rows = [3, 7, 0, 9]
    out, idx, w, _ = orc.layer_rows(rows, shape, x, None, None, Wg, Wu, Wd, Sg, Su, Sd,
                                    router=orc.ROUTER_HASH, token_ids=tok)
    i2, w2 = orc.hash_route(tok[rows], 8, 4, 4, 2)
    np.testing.assert_array_equal(idx, i2)
    np.testing.assert_array_equal(w, w2)
    want = np.stack([orc.shared_row(x[t], Sg, Su, Sd) + sum(
        0.25 * orc.ffn_row(x[t], Wg[idx[r, j]], Wu[idx[r, j]], Wd[idx[r, j]]) for j in range(4))
        for r, t in enumerate(rows)])
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- bias update
def test_bias_update_hand_worked():
    """E = 4, T = 4, K = 2: mean load 2; counts 3, 2, 1, 2 -> down, stay, up, stay."""
    import oracle
    b = oracle.bias_update([3, 2, 1, 2], 4, 2, 0.25, np.array([0.5, -1.0, 0.0, 2.0], np.float32))
    np.testing.assert_array_equal(b, np.array([0.25, -1.0, 0.25, 2.0], np.float32))


def test_bias_update_fractional_mean():
    """E = 3, T = 2, K = 2: mean 4/3, so no expert sits at the mean."""
    import oracle
    b = oracle.bias_update([2, 1, 1], 2, 2, 0.5, np.zeros(3, np.float32))
    np.testing.assert_array_equal(b, np.array([-0.5, 0.5, 0.5], np.float32))


def test_bias_update_mean_compare_is_exact_in_integers():
    """T*K/E with T*K near 2^31: counts at the mean exactly do not move, one off does.
    (A float32 mean would round to a multiple of 64 and misclassify neighbours.)"""
    import oracle
    E, T, K = 3, 2**28 - 2, 8  # T*K = 2^31 - 16, mean 715827877.33
    total = T * K
    assert total % E != 0
    c = total // E
    counts = [c, c + 1, total - 2 * c - 1]
    b = oracle.bias_update(counts, T, K, 1.0, np.zeros(3, np.float32))
    want = [np.sign(total - x * E) for x in counts]
    np.testing.assert_array_equal(b, np.array(want, np.float32))
    E2, T2 = 4, 2**27  # T2*K divisible by E2: mean is exact
    m = T2 * K // E2
    b2 = oracle.bias_update([m, m - 1, m + 1, m], T2, K, 2.0, np.ones(4, np.float32))
    np.testing.assert_array_equal(b2, np.array([1.0, 3.0, -1.0, 1.0], np.float32))


def test_bias_update_is_one_fp32_add():
    import oracle
    bias = np.array([1.0, 1.0, 1e8, -3.0], np.float32)
    g = np.float32(1e-8)
    b = oracle.bias_update([0, 10, 0, 10], 5, 2, float(g), bias)  # mean 2.5
    want = np.array([bias[0] + g, bias[1] - g, bias[2] + g, bias[3] - g], np.float32)
    np.testing.assert_array_equal(b, want)
    assert b[0] == np.float32(1.0) and b[2] == np.float32(1e8)  # rounded away
    b0 = oracle.bias_update([0, 10, 0, 10], 5, 2, 0.0, bias)
    np.testing.assert_array_equal(b0, bias)
