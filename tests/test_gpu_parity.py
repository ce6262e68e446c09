"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Bars (the layer's stated tolerances):
  * selection, gate weights, counts, offsets, send matrices and permutation:
    bit-exact given the same fp32 affinities / the same routing;
  * fp32 router affinities: within 1e-5 absolute;
  * layer output (bf16 inputs, fp32 accumulation, bf16 output): relative
    Frobenius error <= 5e-3 and per-element |err| <= 2e-2 * max |ref|.
Inputs come from the seeded generator (``synth``) only; no expected value is
computed by the CUDA path.
"""
import gc

import numpy as np
import pytest
import torch

import synth
from tests import harness as H

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import combine_expert_ffn_b200 as moe
else:  # collected on CPU-only machines, skipped by the marker filter
    moe = None

DEV = "cuda"


@pytest.fixture(autouse=True)
def _free_gpu():
    yield
    gc.collect()
    torch.cuda.empty_cache()


_cache = {}


def inputs(name):
    """Device inputs of a workload; one large workload cached at a time."""
    if name not in _cache:
        _cache.clear()
        gc.collect()
        torch.cuda.empty_cache()
        _cache[name] = synth.make_inputs(H.shape(name), DEV)
    return _cache[name]


def _i32(*shape):
    return torch.empty(*shape, dtype=torch.int32, device=DEV)


def _f32(*shape):
    return torch.empty(*shape, dtype=torch.float32, device=DEV)


def _bf16(*shape):
    return torch.empty(*shape, dtype=torch.bfloat16, device=DEV)


# ---------------------------------------------------------------- device waits
def test_bounded_wait_times_out_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    moe.moe_selftest_bounded_wait(5_000_000, ws)          # 5 ms limit
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_DEVICE_TIMEOUT
    assert moe.moe_last_device_status(ws) == moe.MOE_ERR_DEVICE_TIMEOUT
    moe.moe_clear_device_status(ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    assert moe.moe_last_device_status(ws) == moe.MOE_OK
    a = torch.arange(10, device=DEV)
    assert int((a * 2).sum()) == 90                        # context still usable


# ---------------------------------------------------------------- selection
@pytest.mark.parametrize("name", ["tiny", "ragged", "ragged2", "mid", "v3", "skew"])
def test_route_select_bit_exact(orc, name):
    sh = H.shape(name)
    scores = synth.uniform01(sh.seed, synth.TENSOR_IDS["scores"], (sh.T, sh.E), DEV)
    bias = synth.normal(sh.seed, synth.TENSOR_IDS["bias"], (sh.E,), max(sh.bias_sigma, 0.05),
                        torch.float32, DEV)
    idx, w = _i32(sh.T, sh.K), _f32(sh.T, sh.K)
    moe.moe_route_select(moe.MoeConfig.of(sh), scores, bias, idx, w)
    ref_idx, ref_w = orc.select(scores.cpu(), bias.cpu(), sh.G, sh.K, sh.M)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_array_equal(w.cpu().numpy().view(np.uint32), ref_w.view(np.uint32))


@pytest.mark.parametrize("E,G,K,M", [(16, 4, 4, 2), (64, 8, 8, 4), (256, 8, 8, 4), (96, 32, 4, 4)])
def test_route_select_exact_ties(orc, E, G, K, M):
    T = 512
    levels = torch.tensor([0.125, 0.25, 0.375, 0.5], device=DEV)
    r = synth.uniform01(11, 99, (T, E), DEV)
    scores = levels[(r * 4).long().clamp(max=3)]
    bias = levels[(synth.uniform01(12, 99, (E,), DEV) * 2).long()] - 0.125
    cfg = moe.MoeConfig(T=T, d=64, E=E, G=G, K=K, M=M, d_ff=64, n_shared=0, d_ff_shared=0)
    idx, w = _i32(T, K), _f32(T, K)
    moe.moe_route_select(cfg, scores, bias, idx, w)
    ref_idx, ref_w = orc.select(scores.cpu(), bias.cpu(), G, K, M)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_array_equal(w.cpu().numpy().view(np.uint32), ref_w.view(np.uint32))


@pytest.mark.parametrize("name,n_sample", [("tiny", None), ("ragged", None), ("ragged2", None),
                                           ("mid", 256), ("v3", 64), ("decode", None),
                                           ("skew", 64)])
def test_route_affinities_and_selection(orc, name, n_sample):
    """moe_route: affinities within 1e-5 of the oracle's; the selection equals
    the oracle's selection on the kernel's own affinities bit for bit (every
    token), and the oracle's on its own affinities except at certified near
    ties.  These workloads cover the fused router's cluster sizes 1 (tiny,
    ragged, skew), 2 (v3), 4 (mid) and 8 (decode)."""
    sh = H.shape(name)
    inp = inputs(name)
    idx, w, s = _i32(sh.T, sh.K), _f32(sh.T, sh.K), _f32(sh.T, sh.E)
    cfg = moe.MoeConfig.of(sh)
    ws = moe.alloc_workspace(cfg)
    moe.moe_route(cfg, inp["x"], inp["router_w"], inp.get("logit_offset"), inp["bias"], idx, w,
                  scores=s, ws=ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    own_idx, own_w = orc.select(s.cpu(), inp["bias"].cpu(), sh.G, sh.K, sh.M)
    np.testing.assert_array_equal(idx.cpu().numpy(), own_idx)
    np.testing.assert_array_equal(w.cpu().numpy().view(np.uint32), own_w.view(np.uint32))
    # without the affinities output the routing is the same
    idx2, w2 = _i32(sh.T, sh.K), _f32(sh.T, sh.K)
    moe.moe_route(cfg, inp["x"], inp["router_w"], inp.get("logit_offset"), inp["bias"], idx2, w2,
                  scores=None, ws=ws)
    assert torch.equal(idx, idx2) and torch.equal(w.view(torch.int32), w2.view(torch.int32))
    rows = np.arange(sh.T) if n_sample is None else \
        np.unique(np.linspace(0, sh.T - 1, n_sample).astype(np.int64))
    ref_s = orc.router_scores(inp["x"].cpu(), inp["router_w"].cpu(), H.host(inp.get("logit_offset")),
                              rows=rows)
    gs = s.cpu().numpy()[rows]
    assert np.abs(gs - ref_s).max() <= H.TOL_AFFINITY
    ref_idx, _ = orc.select(ref_s, inp["bias"].cpu(), sh.G, sh.K, sh.M)
    gi = idx.cpu().numpy()[rows]
    bias = inp["bias"].cpu().numpy()
    flips = 0
    for r in range(len(rows)):
        if not np.array_equal(gi[r], ref_idx[r]):
            flips += 1
            assert H.near_tie_certified(sh, ref_s[r], bias, gi[r], ref_idx[r]), (rows[r], gi[r], ref_idx[r])
    assert flips <= max(1, len(rows) // 100)
    # invariants on every token
    all_idx = idx.cpu().numpy()
    gsz = sh.E // sh.G
    assert ((all_idx >= 0) & (all_idx < sh.E)).all()
    for t in range(0, sh.T, max(1, sh.T // 2048)):
        assert len(set(all_idx[t].tolist())) == sh.K
        assert len({int(e) // gsz for e in all_idx[t]}) <= sh.M
    wsum = w.double().sum(dim=1).cpu().numpy()
    assert np.abs(wsum - 1).max() < 1e-6 and (w > 0).all()


@pytest.mark.parametrize("E,G,K,M,T", [(16, 4, 4, 2, 512), (64, 8, 8, 4, 512),
                                       (256, 8, 8, 4, 512), (96, 32, 4, 4, 512),
                                       (256, 8, 8, 4, 128)])
def test_fused_route_exact_ties(orc, E, G, K, M, T):
    """Exact ties inside the fused router: experts share router rows in pairs
    (bit-identical logits) and the bias takes four levels, so biased affinities
    and group scores tie exactly; the kernel's selection must still equal the
    oracle's on the kernel's own affinities, bit for bit."""
    d = 512
    x = synth.normal(5, 1, (T, d), 1.0, torch.bfloat16, DEV)
    base = synth.normal(5, 2, (E // 2, d), d ** -0.5, torch.float32, DEV)
    router_w = base.repeat_interleave(2, dim=0).contiguous()
    levels = torch.tensor([0.0, 0.125, 0.25, 0.375], device=DEV)
    bias = levels[(synth.uniform01(5, 3, (E,), DEV) * 4).long().clamp(max=3)]
    cfg = moe.MoeConfig(T=T, d=d, E=E, G=G, K=K, M=M, d_ff=64, n_shared=0, d_ff_shared=0)
    idx, w, s = _i32(T, K), _f32(T, K), _f32(T, E)
    ws = moe.alloc_workspace(cfg)
    moe.moe_route(cfg, x, router_w, None, bias, idx, w, scores=s, ws=ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    sh_ = s.cpu()
    assert torch.equal(sh_[:, 0::2].view(torch.int32), sh_[:, 1::2].view(torch.int32))
    ref_idx, ref_w = orc.select(sh_, bias.cpu(), G, K, M)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_array_equal(w.cpu().numpy().view(np.uint32), ref_w.view(np.uint32))


# ---------------------------------------------------------------- dispatch
def _dispatch_gpu(sh, x, topk_idx, with_x=True):
    cfg = moe.MoeConfig.of(sh)
    ws = moe.alloc_workspace(cfg)
    out = {"counts": _i32(sh.E), "offsets": _i32(sh.E + 1), "send": _i32(sh.G, sh.G),
           "send_tok": _i32(sh.G, sh.G), "perm_token": _i32(sh.T * sh.K),
           "inv_perm": _i32(sh.T, sh.K)}
    x_perm = _bf16(sh.T * sh.K, sh.d) if with_x else None
    moe.moe_dispatch(cfg, x, topk_idx, out["counts"], out["offsets"], out["send"], out["send_tok"],
                     out["perm_token"], out["inv_perm"], x_perm, ws)
    status = moe.moe_read_device_status(ws)
    return out, x_perm, status


@pytest.mark.parametrize("name,zipf", [("tiny", 0.0), ("ragged", 1.2), ("ragged2", 0.0),
                                       ("mid", 0.0), ("v3", 0.0), ("skew", 1.2)])
def test_dispatch_bit_exact(orc, name, zipf):
    sh = H.shape(name)
    topk = synth.random_routing(sh.seed, sh.T, sh.E, sh.K, zipf, DEV)
    x = synth.normal(sh.seed, synth.TENSOR_IDS["x"], (sh.T, sh.d), 1.0, torch.bfloat16, DEV)
    out, x_perm, status = _dispatch_gpu(sh, x, topk)
    assert status == moe.MOE_OK
    ref = orc.dispatch(topk.cpu(), sh.E, sh.G)
    for k in ("counts", "offsets", "send", "send_tok", "perm_token", "inv_perm"):
        np.testing.assert_array_equal(out[k].cpu().numpy().reshape(ref[k].shape), ref[k], err_msg=k)
    # x_perm rows are exact copies of the oracle-permuted x rows
    pt = torch.from_numpy(ref["perm_token"].astype(np.int64)).to(DEV)
    assert torch.equal(x_perm.view(torch.int16), x.view(torch.int16)[pt])


@pytest.mark.parametrize("name", ["ragged", "v3"])
def test_permute_alone_equals_dispatch_gather(name):
    """moe_dispatch(x_perm=NULL) + moe_permute == moe_dispatch(x_perm), bit for bit."""
    sh = H.shape(name)
    topk = synth.random_routing(sh.seed, sh.T, sh.E, sh.K, 0.0, DEV)
    x = synth.normal(sh.seed, synth.TENSOR_IDS["x"], (sh.T, sh.d), 1.0, torch.bfloat16, DEV)
    out, x_perm, status = _dispatch_gpu(sh, x, topk)
    assert status == moe.MOE_OK
    out2, none, status = _dispatch_gpu(sh, x, topk, with_x=False)
    assert status == moe.MOE_OK and none is None
    x_perm2 = torch.zeros_like(x_perm)
    moe.moe_permute(moe.MoeConfig.of(sh), x, out2["inv_perm"], x_perm2)
    assert torch.equal(x_perm.view(torch.int16), x_perm2.view(torch.int16))


def test_dispatch_edge_cases(orc):
    # all tokens to the same K experts (one group), T not a multiple of 256
    sh = H.RAGGED.replace(T=300, G=4)
    topk = torch.arange(sh.K, dtype=torch.int32, device=DEV).repeat(sh.T, 1)
    x = synth.normal(1, 1, (sh.T, sh.d), 1.0, torch.bfloat16, DEV)
    out, x_perm, status = _dispatch_gpu(sh, x, topk)
    assert status == moe.MOE_OK
    ref = orc.dispatch(topk.cpu(), sh.E, sh.G)
    for k in ref:
        np.testing.assert_array_equal(out[k].cpu().numpy().reshape(ref[k].shape), ref[k], err_msg=k)


def test_dispatch_flags_bad_ids():
    sh = H.RAGGED.replace(T=8, G=4)
    x = synth.normal(1, 1, (sh.T, sh.d), 1.0, torch.bfloat16, DEV)
    topk = torch.tensor([[0, 1, 2, 3]] * 8, dtype=torch.int32, device=DEV)
    topk[3, 2] = sh.E + 5      # out of range
    _, _, status = _dispatch_gpu(sh, x, topk)
    assert status == moe.MOE_ERR_DEVICE_FAULT
    topk[3, 2] = 1             # repeated expert within a token
    _, _, status = _dispatch_gpu(sh, x, topk)
    assert status == moe.MOE_ERR_DEVICE_FAULT


# ---------------------------------------------------------------- expert FFN
def _ffn_case(orc, sh, counts, seed=0, check_rows=None):
    """Runs moe_expert_ffn on generated x_perm rows with the given segment sizes."""
    counts = np.asarray(counts, np.int64)
    assert len(counts) == sh.E and counts.sum() == sh.T * sh.K
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    n = sh.T * sh.K
    ff, ns, ffs = sh.d_ff, sh.n_shared, sh.d_ff_shared
    x_perm = synth.normal(seed, 21, (n, sh.d), 1.0, torch.bfloat16, DEV)
    x = synth.normal(seed, 22, (sh.T, sh.d), 1.0, torch.bfloat16, DEV)
    wg = synth.normal(seed, 23, (sh.E, ff, sh.d), sh.d ** -0.5, torch.bfloat16, DEV)
    wu = synth.normal(seed, 24, (sh.E, ff, sh.d), sh.d ** -0.5, torch.bfloat16, DEV)
    wd = synth.normal(seed, 25, (sh.E, sh.d, ff), ff ** -0.5, torch.bfloat16, DEV)
    sg = synth.normal(seed, 26, (max(ns, 1), max(ffs, 64), sh.d), sh.d ** -0.5, torch.bfloat16, DEV)
    su = synth.normal(seed, 27, (max(ns, 1), max(ffs, 64), sh.d), sh.d ** -0.5, torch.bfloat16, DEV)
    sd = synth.normal(seed, 28, (max(ns, 1), sh.d, max(ffs, 64)), max(ffs, 64) ** -0.5, torch.bfloat16, DEV)
    y_perm = torch.full((n, sh.d), float("nan"), dtype=torch.bfloat16, device=DEV)
    y_sh = torch.full((sh.T, sh.d), float("nan"), dtype=torch.bfloat16, device=DEV) if ns else None
    cfg = moe.MoeConfig.of(sh)
    ws = moe.alloc_workspace(cfg)
    moe.moe_expert_ffn(cfg, x_perm, torch.from_numpy(offsets).to(DEV), wg, wu, wd, y_perm,
                       x if ns else None, sg if ns else None, su if ns else None,
                       sd if ns else None, y_sh, ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    rows = range(n) if check_rows is None else check_rows
    expert_of = np.searchsorted(offsets, np.arange(n), side="right") - 1
    xh, wgh, wuh, wdh = x_perm.cpu(), wg.cpu(), wu.cpu(), wd.cpu()
    ref = np.stack([orc.ffn_row(xh[r], wgh[expert_of[r]], wuh[expert_of[r]], wdh[expert_of[r]])
                    for r in rows])
    frob, elem = H.compare_out(y_perm[list(rows)], ref)
    assert frob <= H.TOL_FROB and elem <= H.TOL_ELEM, (frob, elem)
    if ns:
        trows = range(sh.T) if check_rows is None else range(0, sh.T, max(1, sh.T // 64))
        xs = x.cpu()
        ref_s = np.stack([orc.shared_row(xs[t], sg.cpu(), su.cpu(), sd.cpu()) for t in trows])
        frob, elem = H.compare_out(y_sh[list(trows)], ref_s)
        assert frob <= H.TOL_FROB and elem <= H.TOL_ELEM, ("shared", frob, elem)


def test_expert_ffn_single_tile(orc):
    sh = synth.MoeShape("one", T=128, d=64, E=1, G=1, K=1, M=1, d_ff=128, n_shared=0,
                        d_ff_shared=0, x_sigma=1, e_sigma=1, bias_sigma=0)
    _ffn_case(orc, sh, [128])


def test_expert_ffn_segment_edges(orc):
    # segment lengths 0, 1, 127, 128, 129, 255, 256, 257 and a long one; 3 row tiles of shared
    counts = [0, 1, 127, 128, 129, 255, 256, 257, 0, 1000]
    sh = synth.MoeShape("edges", T=sum(counts), d=192, E=len(counts), G=1, K=1, M=1, d_ff=192,
                        n_shared=1, d_ff_shared=192, x_sigma=1, e_sigma=1, bias_sigma=0)
    _ffn_case(orc, sh, counts)


def test_expert_ffn_paired_tiles(orc):
    """Experts averaging >= 512 rows take the paired gate/up GEMM (two row tiles
    per weight stage, tiles handed out dynamically): segments that end in a
    full pair, a pair with a 1-row second tile, and a trailing single tile,
    every row against the oracle."""
    counts = [0, 1, 129, 257, 384, 640, 1000, 1023, 1046, 1386]
    sh = synth.MoeShape("pairs", T=sum(counts), d=192, E=len(counts), G=1, K=1, M=1, d_ff=192,
                        n_shared=1, d_ff_shared=192, x_sigma=1, e_sigma=1, bias_sigma=0)
    assert sh.T * sh.K >= 512 * sh.E
    _ffn_case(orc, sh, counts)


def test_expert_ffn_flags_bad_offsets():
    """Offsets outside the buffer or decreasing are reported; nothing is written out of bounds."""
    sh = H.RAGGED2.replace(T=64, n_shared=0, d_ff_shared=0)
    cfg = moe.MoeConfig.of(sh)
    n = sh.T * sh.K
    x_perm = synth.normal(1, 21, (n, sh.d), 1.0, torch.bfloat16, DEV)
    wg = synth.normal(1, 23, (sh.E, sh.d_ff, sh.d), 0.1, torch.bfloat16, DEV)
    wd = synth.normal(1, 25, (sh.E, sh.d, sh.d_ff), 0.1, torch.bfloat16, DEV)
    offsets = torch.linspace(0, n, sh.E + 1, device=DEV).to(torch.int32)
    offsets[7] = offsets[9] + 5          # a decreasing pair
    guard = torch.zeros(n + 64, sh.d, dtype=torch.bfloat16, device=DEV)
    y_perm = guard[:n]
    ws = moe.alloc_workspace(cfg)
    moe.moe_expert_ffn(cfg, x_perm, offsets, wg, wg, wd, y_perm, None, None, None, None, None, ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_DEVICE_FAULT
    assert int(guard[n:].view(torch.int16).abs().sum()) == 0   # the tail guard is untouched


@pytest.mark.parametrize("name", ["ragged", "ragged2", "noshared", "tiny"])
def test_expert_ffn_ragged(orc, name):
    sh = H.shape(name)
    topk = synth.random_routing(sh.seed, sh.T, sh.E, sh.K, 1.0, "cpu")
    counts = np.bincount(topk.numpy().ravel(), minlength=sh.E)
    _ffn_case(orc, sh, counts, seed=sh.seed)


# ---------------------------------------------------------------- combine
@pytest.mark.parametrize("name", ["tiny", "ragged2", "mid"])
def test_combine(orc, name):
    sh = H.shape(name)
    topk = synth.random_routing(sh.seed, sh.T, sh.E, sh.K, 0.0, "cpu")
    ref_d = orc.dispatch(topk, sh.E, sh.G)
    w = synth.uniform01(sh.seed, 31, (sh.T, sh.K))
    w = (w / w.sum(dim=1, keepdim=True)).float()
    y_perm = synth.normal(sh.seed, synth.TENSOR_IDS["y_perm"], (sh.T * sh.K, sh.d), 1.0)
    y_sh = synth.normal(sh.seed, synth.TENSOR_IDS["y_shared"], (sh.T, sh.d), 1.0)
    inv = torch.from_numpy(ref_d["inv_perm"])
    out = _bf16(sh.T, sh.d)
    cfg = moe.MoeConfig.of(sh)
    moe.moe_combine(cfg, y_perm.to(DEV), inv.to(DEV), w.to(DEV), y_sh.to(DEV), out)
    ref = orc.combine(y_perm, inv, w, y_sh)
    frob, elem = H.compare_out(out, ref)
    assert frob <= 4e-3 and elem <= 8e-3, (frob, elem)
    out0 = _bf16(sh.T, sh.d)
    moe.moe_combine(cfg, y_perm.to(DEV), inv.to(DEV), w.to(DEV), None, out0)
    frob, elem = H.compare_out(out0, orc.combine(y_perm, inv, w, None))
    assert frob <= 4e-3 and elem <= 8e-3, (frob, elem)


# ---------------------------------------------------------------- whole layer
def _forward(sh, inp):
    cfg = moe.MoeConfig.of(sh)
    ws = moe.alloc_workspace(cfg)
    o = moe.forward_outputs(cfg)
    moe.moe_forward(cfg, inp["x"], inp["router_w"], inp.get("logit_offset"), inp["bias"],
                    inp["w_gate"], inp["w_up"], inp["w_down"], inp.get("ws_gate"),
                    inp.get("ws_up"), inp.get("ws_down"), o["out"], o["topk_idx"], o["topk_w"],
                    o["counts"], o["offsets"], o["send"], o["send_tok"], ws=ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    return o


def _check_plan_properties(sh, o):
    idx = o["topk_idx"].cpu().numpy()
    counts = o["counts"].cpu().numpy()
    offsets = o["offsets"].cpu().numpy()
    send = o["send"].cpu().numpy()
    send_tok = o["send_tok"].cpu().numpy()
    np.testing.assert_array_equal(counts, np.bincount(idx.ravel(), minlength=sh.E))
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    assert send.sum() == sh.T * sh.K
    np.testing.assert_array_equal(send.sum(axis=1), np.full(sh.G, sh.T // sh.G * sh.K))
    gsz = sh.E // sh.G
    np.testing.assert_array_equal(send.sum(axis=0), counts.reshape(sh.G, gsz).sum(axis=1))
    groups_per_token = np.array([len({int(e) // gsz for e in r}) for r in idx])
    assert groups_per_token.max() <= sh.M
    np.testing.assert_array_equal(send_tok.sum(), groups_per_token.sum())


@pytest.mark.parametrize("name,n_sample", [("tiny", None), ("ragged", None), ("ragged2", None),
                                           ("noshared", None), ("mid", 256), ("v3", 256),
                                           ("decode", None), ("skew", 256)])
def test_forward_matches_oracle(orc, name, n_sample):
    """Whole layer against the oracle: every token of the small workloads and of
    the decode batch; at the large ones a spread of tokens plus the tokens in the
    last row tiles of the most-loaded experts and at the highest x_perm rows
    (above the 2^31-byte offset at skew), run on every host core."""
    sh = H.shape(name)
    inp = inputs(name)
    o = _forward(sh, inp)
    _check_plan_properties(sh, o)
    gi_all = o["topk_idx"].cpu().numpy()
    rows = np.arange(sh.T) if n_sample is None else H.parity_rows(sh, gi_all, n_spread=n_sample)
    if n_sample is not None:
        assert len(rows) >= n_sample
    ref_out, ref_idx, ref_w, ref_s = H.oracle_layer_sample(orc, sh, inp, rows,
                                                           threads=orc.all_cores())
    gi = gi_all[rows]
    keep = []
    bias = inp["bias"].cpu().numpy()
    for r in range(len(rows)):
        if np.array_equal(gi[r], ref_idx[r]):
            keep.append(r)
        else:
            assert H.near_tie_certified(sh, ref_s[r], bias, gi[r], ref_idx[r])
    assert len(keep) >= len(rows) - max(1, len(rows) // 100)
    frob, elem = H.compare_out(o["out"][torch.as_tensor(rows[keep], device=DEV)], ref_out[keep])
    assert frob <= H.TOL_FROB and elem <= H.TOL_ELEM, (frob, elem)


def test_forward_zero_tokens():
    sh = H.RAGGED.replace(T=0)
    cfg = moe.MoeConfig.of(sh)
    ws = moe.alloc_workspace(cfg)
    inp = synth.make_inputs(H.RAGGED, DEV)
    out = _bf16(1, sh.d)
    moe.moe_forward(cfg, inp["x"], inp["router_w"], None, inp["bias"], inp["w_gate"], inp["w_up"],
                    inp["w_down"], inp["ws_gate"], inp["ws_up"], inp["ws_down"], out, ws=ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
