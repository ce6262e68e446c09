"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks one step against something independent of the oracle's own
code: a hand-worked example (tests/golden/route_4tok.txt), brute-force
enumeration, a sort-based restatement, a closed form, or a numpy / scipy
library routine.  They are chosen so that a dropped term, a wrong sign or
index, or a transposed operand in the oracle fails at least one of them.
"""
import itertools
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy.special import expit

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "route_4tok.txt")


def _bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _bf16_np(t):
    return t.float().numpy().astype(np.float64)


def load_golden():
    g = {"scores": {}, "topk_idx": {}, "topk_w": {}, "group_score": {}}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            if key in g:
                g[key][int(vals[0])] = vals[1:]
            else:
                g[key] = vals
    return g


# ---------------------------------------------------------------- selection
def test_golden_4token_routing_and_dispatch(orc):
    g = load_golden()
    E, G, K, M = (int(g[k][0]) for k in ("E", "G", "K", "M"))
    T = len(g["scores"])
    scores = np.array([[float(v) for v in g["scores"][t]] for t in range(T)], np.float32)
    bias = np.array([float(v) for v in g["bias"]], np.float32)
    idx, w, gs = orc.select(scores, bias, G, K, M, want_group_score=True)
    for t in range(T):
        assert idx[t].tolist() == [int(v) for v in g["topk_idx"][t]], t
        assert gs[t].tolist() == [float(v) for v in g["group_score"][t]], t
        for j, frac in enumerate(g["topk_w"][t]):
            exact = float(Fraction(frac))
            assert abs(float(w[t, j]) - exact) <= np.spacing(np.float32(exact)), (t, j)
    disp = orc.dispatch(idx, E, G)
    for key in ("counts", "offsets", "perm_token", "inv_perm", "send", "send_tok"):
        assert disp[key].ravel().tolist() == [int(v) for v in g[key]], key


def _brute_select(b, s, G, K, M):
    """Enumerate every group subset and expert subset (distinct values only)."""
    E = len(b)
    gsz, kpg = E // G, K // M
    gscore = []
    for gi in range(G):
        mem = range(gi * gsz, (gi + 1) * gsz)
        gscore.append(max(sum(float(b[i]) for i in c) for c in itertools.combinations(mem, kpg)))
    best_groups = max(itertools.combinations(range(G), M), key=lambda c: sum(gscore[q] for q in c))
    allowed = [i for i in range(E) if i // gsz in best_groups]
    best = max(itertools.combinations(allowed, K), key=lambda c: sum(float(b[i]) for i in c))
    return set(best), set(best_groups)


@pytest.mark.parametrize("E,G,K,M", [(8, 2, 2, 1), (8, 4, 4, 2), (12, 3, 4, 2), (16, 4, 4, 2),
                                     (16, 4, 6, 2), (16, 8, 3, 3), (16, 2, 4, 1)])
def test_select_matches_bruteforce_enumeration(orc, E, G, K, M):
    rng = np.random.default_rng(E * 100 + G * 10 + K + M)
    for trial in range(40):
        s = rng.uniform(0.01, 0.99, size=(1, E)).astype(np.float32)
        bias = rng.normal(0, 0.1, size=E).astype(np.float32)
        b = (s[0] + bias).astype(np.float32)
        if len(set(b.tolist())) < E:
            continue
        idx, w = orc.select(s, bias, G, K, M)
        want, groups = _brute_select(b, s[0], G, K, M)
        assert set(idx[0].tolist()) == want, (trial, idx, want)
        assert {i // (E // G) for i in idx[0]} <= groups
        # descending biased affinity
        assert all(b[idx[0][j]] > b[idx[0][j + 1]] for j in range(K - 1))
        # weights use the UNBIASED affinities
        ref = s[0][idx[0]].astype(np.float64) / s[0][idx[0]].astype(np.float64).sum()
        np.testing.assert_allclose(w[0], ref, rtol=2e-7, atol=0)


def _sorted_select(s, bias, G, K, M):
    """Restatement by sorting with key (-value, index): the canonical tie rule."""
    E = len(s)
    gsz, kpg = E // G, K // M
    b = (np.asarray(s, np.float32) + np.asarray(bias, np.float32)).astype(np.float32)
    gscore = []
    for gi in range(G):
        mem = sorted(range(gi * gsz, (gi + 1) * gsz), key=lambda i: (-b[i], i))[:kpg]
        acc = np.float32(b[mem[0]])
        for i in mem[1:]:
            acc = np.float32(acc + b[i])
        gscore.append(acc)
    keep = sorted(range(G), key=lambda q: (-gscore[q], q))[:M]
    allowed = [i for i in range(E) if i // gsz in keep]
    return sorted(allowed, key=lambda i: (-b[i], i))[:K], gscore


@pytest.mark.parametrize("E,G,K,M", [(16, 4, 4, 2), (32, 8, 6, 3), (64, 8, 8, 4), (256, 8, 8, 4)])
def test_select_ties_follow_lower_index_rule(orc, E, G, K, M):
    rng = np.random.default_rng(7 + E)
    levels = np.array([0.125, 0.25, 0.375, 0.5], np.float32)  # heavy exact ties
    s = levels[rng.integers(0, 4, size=(64, E))]
    bias = levels[rng.integers(0, 2, size=E)] - np.float32(0.125)
    idx, w, gs = orc.select(s, bias, G, K, M, want_group_score=True)
    for t in range(64):
        want, gscore = _sorted_select(s[t], bias, G, K, M)
        assert idx[t].tolist() == want, t
        assert gs[t].tolist() == [float(v) for v in gscore]


def test_select_invariants_v3_shape(orc):
    shape = synth.config("v3")
    E, G, K, M = shape.E, shape.G, shape.K, shape.M
    rng = np.random.default_rng(3)
    s = expit(rng.normal(0, 1, size=(512, E))).astype(np.float32)
    bias = rng.normal(0, 0.5, size=E).astype(np.float32)
    idx, w, gs = orc.select(s, bias, G, K, M, want_group_score=True)
    gsz = E // G
    for t in range(512):
        row = idx[t].tolist()
        assert len(set(row)) == K
        groups = {i // gsz for i in row}
        assert len(groups) <= M                      # the node limit holds
        top_groups = set(sorted(range(G), key=lambda q: (-gs[t][q], q))[:M])
        assert groups <= top_groups
        assert abs(float(np.float64(w[t]).sum()) - 1.0) < 1e-6
        assert (w[t] > 0).all()


# ---------------------------------------------------------------- dispatch
@pytest.mark.parametrize("T,E,G,K", [(64, 16, 4, 4), (96, 32, 8, 6), (1000, 64, 8, 8)])
def test_dispatch_matches_stable_argsort(orc, T, E, G, K):
    rng = np.random.default_rng(T)
    idx = np.stack([rng.choice(E, size=K, replace=False) for _ in range(T)]).astype(np.int32)
    out = orc.dispatch(idx, E, G)
    flat = idx.ravel()
    order = np.argsort(flat, kind="stable")          # copies sorted by expert, (t,j) order kept
    np.testing.assert_array_equal(out["perm_token"], order // K)
    inv = np.empty(T * K, np.int64)
    inv[order] = np.arange(T * K)
    np.testing.assert_array_equal(out["inv_perm"].ravel(), inv)
    np.testing.assert_array_equal(out["counts"], np.bincount(flat, minlength=E))
    np.testing.assert_array_equal(out["offsets"], np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
    send = np.zeros((G, G), np.int64)
    src = np.repeat(np.arange(T) // (T // G), K)
    np.add.at(send, (src, flat // (E // G)), 1)
    np.testing.assert_array_equal(out["send"], send)
    send_tok = np.zeros((G, G), np.int64)
    for t in range(T):
        for g in set((idx[t] // (E // G)).tolist()):
            send_tok[t // (T // G), g] += 1
    np.testing.assert_array_equal(out["send_tok"], send_tok)
    assert out["send"].sum() == T * K
    assert (out["send_tok"].sum(axis=1) <= (T // G) * K).all()
    # permutation followed by its inverse is the identity
    np.testing.assert_array_equal(out["perm_token"][out["inv_perm"].ravel()], np.repeat(np.arange(T), K))


def test_dispatch_rejects_bad_routing(orc):
    with pytest.raises(ValueError):
        orc.dispatch(np.array([[0, 16]], np.int32), 16, 1)
    with pytest.raises(ValueError):
        orc.dispatch(np.array([[3, 3]], np.int32), 16, 1)


# ---------------------------------------------------------------- router
def test_router_zero_weights_give_one_half(orc):
    x = _bf16(np.random.default_rng(0).normal(size=(5, 64)))
    s = orc.router_scores(x, np.zeros((8, 64), np.float32))
    assert (s == 0.5).all()


def test_router_one_hot_weights_pick_the_right_feature(orc):
    rng = np.random.default_rng(1)
    x = _bf16(rng.normal(size=(6, 16)))
    e = np.zeros((5, 16), np.float32)
    for i in range(5):
        e[i, 3 * i + 1] = 1.0
    s = orc.router_scores(x, e)
    xs = _bf16_np(x)
    want = expit(xs[:, [1, 4, 7, 10, 13]]).astype(np.float32)
    np.testing.assert_array_equal(s, want)


def test_router_random_against_numpy_matmul(orc):
    rng = np.random.default_rng(2)
    x = _bf16(rng.normal(size=(33, 96)))
    e = rng.normal(0, 0.1, size=(20, 96)).astype(np.float32)
    off = rng.normal(0, 1, size=20).astype(np.float32)
    s = orc.router_scores(x, e, off)
    L = _bf16_np(x) @ e.astype(np.float64).T + off.astype(np.float64)
    np.testing.assert_allclose(s, expit(L), rtol=0, atol=1e-7)
    rows = [5, 0, 32]
    np.testing.assert_array_equal(orc.router_scores(x, e, off, rows=rows), s[rows])


# ---------------------------------------------------------------- FFN / combine
def _swiglu_np(x, Wg, Wu, Wd):
    u = x @ Wg.T
    v = x @ Wu.T
    return (u * expit(u) * v) @ Wd.T


def test_ffn_identity_weights_closed_form(orc):
    """W_g = a I, W_u = c I, W_d = I  =>  y_k = SiLU(a x_k) * (c x_k)."""
    d, a, c = 32, 0.5, 2.0
    x = _bf16(np.random.default_rng(4).normal(size=d))
    Wg = _bf16(a * np.eye(d))
    Wu = _bf16(c * np.eye(d))
    Wd = _bf16(np.eye(d))
    y = orc.ffn_row(x, Wg, Wu, Wd)
    xs = _bf16_np(x)
    np.testing.assert_allclose(y, (a * xs) * expit(a * xs) * (c * xs), rtol=1e-14, atol=1e-15)


def test_ffn_row_against_numpy_swiglu(orc):
    rng = np.random.default_rng(5)
    d, f = 48, 24                               # non-square: a transposed operand fails
    x = _bf16(rng.normal(size=d))
    Wg, Wu, Wd = _bf16(rng.normal(size=(f, d)) / 7), _bf16(rng.normal(size=(f, d)) / 7), _bf16(rng.normal(size=(d, f)) / 5)
    y = orc.ffn_row(x, Wg, Wu, Wd)
    want = _swiglu_np(_bf16_np(x), _bf16_np(Wg), _bf16_np(Wu), _bf16_np(Wd))
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-14)
    # shared experts: n_shared FFNs summed
    Wsg = torch.stack([Wg, _bf16(rng.normal(size=(f, d)) / 7)])
    Wsu = torch.stack([Wu, _bf16(rng.normal(size=(f, d)) / 7)])
    Wsd = torch.stack([Wd, _bf16(rng.normal(size=(d, f)) / 5)])
    ys = orc.shared_row(x, Wsg, Wsu, Wsd)
    want2 = sum(_swiglu_np(_bf16_np(x), _bf16_np(Wsg[i]), _bf16_np(Wsu[i]), _bf16_np(Wsd[i])) for i in range(2))
    np.testing.assert_allclose(ys, want2, rtol=1e-12, atol=1e-14)


def _layer_inputs(shape, rng, identical=False):
    E, d, ff = shape.E, shape.d, shape.d_ff
    x = _bf16(rng.normal(size=(shape.T, d)))
    e = rng.normal(0, 0.3, size=(E, d)).astype(np.float32)
    mk = lambda *s: _bf16(rng.normal(size=s) / np.sqrt(s[-1]))
    if identical:
        g, u, dn = mk(ff, d), mk(ff, d), mk(d, ff)
        Wg, Wu, Wd = [g] * E, [u] * E, [dn] * E
    else:
        Wg = [mk(ff, d) for _ in range(E)]
        Wu = [mk(ff, d) for _ in range(E)]
        Wd = [mk(d, ff) for _ in range(E)]
    ns, ffs = shape.n_shared, shape.d_ff_shared
    Ws = (torch.stack([mk(ffs, d) for _ in range(ns)]), torch.stack([mk(ffs, d) for _ in range(ns)]),
          torch.stack([mk(d, ffs) for _ in range(ns)]))
    return x, e, Wg, Wu, Wd, Ws


def test_layer_single_expert_is_plain_swiglu(orc):
    """E = G = K = M = 1: the layer is FFN_0(x) + shared(x) with gate weight 1."""
    shape = synth.MoeShape("one", T=6, d=40, E=1, G=1, K=1, M=1, d_ff=24, n_shared=1,
                           d_ff_shared=16, x_sigma=1, e_sigma=1, bias_sigma=0)
    rng = np.random.default_rng(6)
    x, e, Wg, Wu, Wd, (Sg, Su, Sd) = _layer_inputs(shape, rng)
    out, idx, w, _ = orc.layer_rows(range(6), shape, x, e, np.zeros(1, np.float32),
                                    Wg, Wu, Wd, Sg, Su, Sd)
    assert (idx == 0).all() and (w == 1.0).all()
    xs = _bf16_np(x)
    want = _swiglu_np(xs, _bf16_np(Wg[0]), _bf16_np(Wu[0]), _bf16_np(Wd[0])) + \
        _swiglu_np(xs, _bf16_np(Sg[0]), _bf16_np(Su[0]), _bf16_np(Sd[0]))
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-13)


def test_layer_identical_experts_is_routing_independent(orc):
    """All routed experts equal  =>  out = FFN(x) * sum_j w_j + shared = FFN(x) + shared."""
    shape = synth.MoeShape("same", T=16, d=32, E=16, G=4, K=4, M=2, d_ff=24, n_shared=2,
                           d_ff_shared=8, x_sigma=1, e_sigma=1, bias_sigma=0)
    rng = np.random.default_rng(8)
    x, e, Wg, Wu, Wd, (Sg, Su, Sd) = _layer_inputs(shape, rng, identical=True)
    outs = []
    for bias_seed in (0, 1):
        bias = np.random.default_rng(bias_seed).normal(0, 2, size=16).astype(np.float32)
        out, idx, _, _ = orc.layer_rows(range(16), shape, x, e, bias, Wg, Wu, Wd, Sg, Su, Sd)
        outs.append((out, idx))
    assert not np.array_equal(outs[0][1], outs[1][1])          # routings differ ...
    # ... outputs do not (up to the fp32 rounding of sum_j w_j = 1)
    np.testing.assert_allclose(outs[0][0], outs[1][0], rtol=1e-6, atol=1e-6)
    xs = _bf16_np(x)
    want = _swiglu_np(xs, _bf16_np(Wg[0]), _bf16_np(Wu[0]), _bf16_np(Wd[0])) + sum(
        _swiglu_np(xs, _bf16_np(Sg[i]), _bf16_np(Su[i]), _bf16_np(Sd[i])) for i in range(2))
    np.testing.assert_allclose(outs[0][0], want, rtol=1e-6, atol=1e-7)


def test_layer_rows_equals_composed_steps(orc):
    """Whole-layer entry = scores -> select -> dispatch -> per-row FFN -> combine (numpy gather)."""
    shape = synth.MoeShape("mini", T=24, d=32, E=8, G=4, K=4, M=2, d_ff=16, n_shared=1,
                           d_ff_shared=8, x_sigma=1, e_sigma=1, bias_sigma=0.1)
    rng = np.random.default_rng(9)
    x, e, Wg, Wu, Wd, (Sg, Su, Sd) = _layer_inputs(shape, rng)
    bias = rng.normal(0, 0.1, size=8).astype(np.float32)
    out, idx, w, sc = orc.layer_rows(range(24), shape, x, e, bias, Wg, Wu, Wd, Sg, Su, Sd)
    disp = orc.dispatch(idx, 8, 4)
    ypf = np.stack([orc.ffn_row(x[t], Wg[ex], Wu[ex], Wd[ex])
                    for ex in range(8) for t in disp["perm_token"][disp["offsets"][ex]:disp["offsets"][ex + 1]]])
    ysh = np.stack([orc.shared_row(x[t], Sg, Su, Sd) for t in range(24)])
    want = ysh + (w[:, :, None].astype(np.float64) * ypf[disp["inv_perm"]]).sum(axis=1)
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-13)


def test_combine_against_numpy_gather(orc):
    rng = np.random.default_rng(10)
    T, K, d = 20, 3, 16
    yp = _bf16(rng.normal(size=(T * K, d)))
    inv = rng.permutation(T * K).reshape(T, K).astype(np.int32)
    w = rng.uniform(0.1, 1, size=(T, K)).astype(np.float32)
    ys = _bf16(rng.normal(size=(T, d)))
    out = orc.combine(yp, inv, w, ys)
    want = _bf16_np(ys) + (w[:, :, None].astype(np.float64) * _bf16_np(yp)[inv]).sum(axis=1)
    np.testing.assert_allclose(out, want, rtol=1e-13, atol=1e-14)
    out0 = orc.combine(yp, inv, w, None)
    np.testing.assert_allclose(out0, want - _bf16_np(ys), rtol=1e-12, atol=1e-13)


def test_round_h_only_perturbs_at_bf16_level(orc):
    rng = np.random.default_rng(11)
    d, f = 64, 32
    x = _bf16(rng.normal(size=d))
    Wg, Wu, Wd = _bf16(rng.normal(size=(f, d)) / 8), _bf16(rng.normal(size=(f, d)) / 8), _bf16(rng.normal(size=(d, f)) / 6)
    y0 = orc.ffn_row(x, Wg, Wu, Wd, round_h=False)
    y1 = orc.ffn_row(x, Wg, Wu, Wd, round_h=True)
    rel = np.linalg.norm(y1 - y0) / np.linalg.norm(y0)
    assert 0 < rel < 8e-3


def test_layer_without_shared_experts(orc):
    """n_shared = 0: the layer is the gate-weighted routed sum alone."""
    shape = synth.MoeShape("nosh", T=8, d=32, E=8, G=4, K=2, M=2, d_ff=16, n_shared=0,
                           d_ff_shared=0, x_sigma=1, e_sigma=1, bias_sigma=0)
    rng = np.random.default_rng(12)
    x, e, Wg, Wu, Wd, _ = _layer_inputs(shape.replace(n_shared=1, d_ff_shared=8), rng)
    bias = np.zeros(8, np.float32)
    empty = torch.zeros(1, 8, 32, dtype=torch.bfloat16)
    out, idx, w, _ = orc.layer_rows(range(8), shape, x, e, bias, Wg, Wu, Wd, empty, empty,
                                    torch.zeros(1, 32, 8, dtype=torch.bfloat16))
    xs = _bf16_np(x)
    want = np.stack([sum(float(w[t, j]) * _swiglu_np(xs[t], _bf16_np(Wg[idx[t, j]]), _bf16_np(Wu[idx[t, j]]),
                                                     _bf16_np(Wd[idx[t, j]])) for j in range(2))
                     for t in range(8)])
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-13)
