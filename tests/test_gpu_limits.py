"""The CUDA path at the edges of the supported sizes and in degenerate layers.

Maximum routing sizes (E = 1024 experts, G = 64 groups, K = 32, M up to 32),
no node limit (M = G), every expert chosen (K = E), the smallest batch
(T = G), and many tiny expert segments.  Bars as in the main parity tests:
selection and dispatch bit-exact, layer output within the output bars; the
layers through the tile-packed weights bit-identical to the row-major ones.
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


def _shape(name, **kw):
    base = dict(x_sigma=1.0, e_sigma=0.1, bias_sigma=0.05, seed=11)
    base.update(kw)
    return synth.MoeShape(name, **base)


MAX_ROUTE = [(1024, 64, 32, 16), (1024, 64, 32, 32), (1024, 8, 32, 4), (1024, 64, 1, 1),
             (64, 64, 32, 32)]


@pytest.mark.parametrize("E,G,K,M", MAX_ROUTE)
def test_route_select_at_max_sizes(orc, E, G, K, M):
    T = 2048
    cfg = moe.MoeConfig(T=T, d=64, E=E, G=G, K=K, M=M, d_ff=64, n_shared=0, d_ff_shared=0)
    scores = synth.uniform01(5, 50, (T, E), DEV)
    bias = synth.normal(5, 51, (E,), 0.05, torch.float32, DEV)
    idx = torch.empty(T, K, dtype=torch.int32, device=DEV)
    w = torch.empty(T, K, dtype=torch.float32, device=DEV)
    moe.moe_route_select(cfg, scores, bias, idx, w)
    ref_idx, ref_w = orc.select(scores.cpu(), bias.cpu(), G, K, M)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_array_equal(w.cpu().numpy().view(np.uint32), ref_w.view(np.uint32))


# 70016 tokens make 274 blocks of 256: more than the scatter kernel sums itself,
# so the separate block-scan kernel runs
@pytest.mark.parametrize("T,E,G,K", [(2048, 1024, 64, 32), (64, 1024, 64, 32), (128, 1024, 1, 1),
                                     (70016, 256, 8, 8)])
def test_dispatch_at_max_sizes(orc, T, E, G, K):
    sh = _shape("dmax", T=T, d=128, E=E, G=G, K=K, M=1 if K == 1 else min(16, G), d_ff=64,
                n_shared=0, d_ff_shared=0)
    topk = synth.random_routing(3, T, E, K, 1.1, DEV)
    x = synth.normal(3, 1, (T, sh.d), 1.0, torch.bfloat16, DEV)
    cfg = moe.MoeConfig.of(sh)
    ws = moe.alloc_workspace(cfg)
    i32 = lambda *s: torch.empty(*s, dtype=torch.int32, device=DEV)  # noqa: E731
    out = {"counts": i32(E), "offsets": i32(E + 1), "send": i32(G, G), "send_tok": i32(G, G),
           "perm_token": i32(T * K), "inv_perm": i32(T, K)}
    x_perm = torch.empty(T * K, sh.d, dtype=torch.bfloat16, device=DEV)
    moe.moe_dispatch(cfg, x, topk, out["counts"], out["offsets"], out["send"], out["send_tok"],
                     out["perm_token"], out["inv_perm"], x_perm, ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    ref = orc.dispatch(topk.cpu(), E, G)
    for k in ref:
        np.testing.assert_array_equal(out[k].cpu().numpy().reshape(ref[k].shape), ref[k], err_msg=k)
    pt = torch.from_numpy(ref["perm_token"].astype(np.int64)).to(DEV)
    assert torch.equal(x_perm.view(torch.int16), x.view(torch.int16)[pt])


LAYERS = [
    # many tiny expert segments: 1024 experts, 32 per token, ~32 rows each
    _shape("max_experts", T=1024, d=128, E=1024, G=64, K=32, M=16, d_ff=64, n_shared=1,
           d_ff_shared=64),
    # no node limit: M = G
    _shape("no_limit", T=256, d=192, E=32, G=4, K=8, M=4, d_ff=128, n_shared=1, d_ff_shared=64),
    # every expert chosen: the gates are s / sum(s) over all experts
    _shape("all_experts", T=128, d=128, E=8, G=2, K=8, M=2, d_ff=64, n_shared=0, d_ff_shared=0),
    # the smallest batch: one token per group
    _shape("t_equals_g", T=8, d=256, E=64, G=8, K=8, M=4, d_ff=128, n_shared=2, d_ff_shared=64),
]


@pytest.mark.parametrize("sh", LAYERS, ids=[s.name for s in LAYERS])
def test_forward_degenerate_and_max_layers(orc, sh):
    inp = synth.make_inputs(sh, DEV)
    cfg = moe.MoeConfig.of(sh)
    ws = moe.alloc_workspace(cfg)
    o = moe.forward_outputs(cfg)
    moe.moe_forward(cfg, inp["x"], inp["router_w"], None, inp["bias"], inp["w_gate"],
                    inp["w_up"], inp["w_down"], inp.get("ws_gate"), inp.get("ws_up"),
                    inp.get("ws_down"), o["out"], o["topk_idx"], o["topk_w"], o["counts"],
                    o["offsets"], o["send"], o["send_tok"], ws=ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    rows = np.arange(sh.T)
    ref_out, ref_idx, _, ref_s = H.oracle_layer_sample(orc, sh, inp, rows)
    gi = o["topk_idx"].cpu().numpy()
    keep = [r for r in rows if np.array_equal(gi[r], ref_idx[r])]
    for r in set(rows.tolist()) - set(keep):
        assert H.near_tie_certified(sh, ref_s[r], inp["bias"].cpu().numpy(), gi[r], ref_idx[r])
    assert len(keep) >= len(rows) - max(1, len(rows) // 100)
    frob, elem = H.compare_out(o["out"][torch.as_tensor(keep, device=DEV)], ref_out[keep])
    assert frob <= H.TOL_FROB and elem <= H.TOL_ELEM, (frob, elem)
    if sh.K == sh.E:
        assert (np.sort(gi, axis=1) == np.arange(sh.E)).all()
    # the tile-packed weights give the same layer bit for bit
    packed = moe.pack_weights(cfg, inp["w_gate"], inp["w_up"], inp["w_down"], inp.get("ws_gate"),
                              inp.get("ws_up"), inp.get("ws_down"))
    o2 = moe.forward_outputs(cfg)
    moe.moe_forward_packed(cfg, inp["x"], inp["router_w"], None, inp["bias"], packed, o2["out"],
                           o2["topk_idx"], o2["topk_w"], o2["counts"], o2["offsets"], o2["send"],
                           o2["send_tok"], ws=ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    assert torch.equal(o2["topk_idx"], o["topk_idx"])
    assert torch.equal(o2["out"].view(torch.int16), o["out"].view(torch.int16))


# Router work split over d (small batches): decode has 2 tiles and 28 k ranges;
# T=640, E=128, d=7040 has 5 tiles and 27 ranges of 5 k blocks, the last five of
# them empty (their partial logits are zeros).
SPLIT_ROUTES = [
    ("decode", None),
    ("split_empty", _shape("split_empty", T=640, d=7040, E=128, G=8, K=8, M=4, d_ff=64,
                           n_shared=0, d_ff_shared=0, x_sigma=1.0, e_sigma=7040 ** -0.5)),
]


@pytest.mark.parametrize("name,sh", SPLIT_ROUTES, ids=[n for n, _ in SPLIT_ROUTES])
@pytest.mark.parametrize("router", [0, 1])
def test_router_split_over_d(orc, name, sh, router):
    sh = H.shape(name) if sh is None else sh
    inp = synth.make_inputs(sh, DEV, weights=False)
    cfg = moe.MoeConfig.of(sh, router=router)
    idx = torch.empty(sh.T, sh.K, dtype=torch.int32, device=DEV)
    w = torch.empty(sh.T, sh.K, dtype=torch.float32, device=DEV)
    s = torch.empty(sh.T, sh.E, dtype=torch.float32, device=DEV)
    ws = moe.alloc_workspace(cfg)
    moe.moe_route(cfg, inp["x"], inp["router_w"], inp.get("logit_offset"), inp["bias"], idx, w,
                  scores=s, ws=ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    rows = np.unique(np.linspace(0, sh.T - 1, 48).astype(np.int64))
    ref = orc.router_scores(inp["x"].cpu(), inp["router_w"].cpu(), H.host(inp.get("logit_offset")),
                            rows=rows, affinity=router)
    gs = s.cpu().numpy()
    assert np.abs(gs[rows] - ref).max() <= H.TOL_AFFINITY
    sel_idx, sel_w = orc.select(gs, inp["bias"].cpu(), sh.G, sh.K, sh.M)
    np.testing.assert_array_equal(idx.cpu().numpy(), sel_idx)
    np.testing.assert_array_equal(w.cpu().numpy().view(np.uint32), sel_w.view(np.uint32))
