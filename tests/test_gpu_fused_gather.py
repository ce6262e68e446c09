"""The expert FFN fused with the dispatch gather (moe_expert_ffn_gather).

Bars: bit-identical to the two-step path (moe_dispatch writing x_perm, then
moe_expert_ffn reading it) on the same routing -- the same bf16 operands meet
the same MMAs in the same order -- and within the layer's output tolerances
of the oracle on the rows it computes.
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


def _weights(sh, seed):
    ff, ns, ffs = sh.d_ff, sh.n_shared, max(sh.d_ff_shared, 64)
    w = {
        "wg": synth.normal(seed, 23, (sh.E, ff, sh.d), sh.d ** -0.5, torch.bfloat16, DEV),
        "wu": synth.normal(seed, 24, (sh.E, ff, sh.d), sh.d ** -0.5, torch.bfloat16, DEV),
        "wd": synth.normal(seed, 25, (sh.E, sh.d, ff), ff ** -0.5, torch.bfloat16, DEV),
    }
    if ns:
        w["sg"] = synth.normal(seed, 26, (ns, ffs, sh.d), sh.d ** -0.5, torch.bfloat16, DEV)
        w["su"] = synth.normal(seed, 27, (ns, ffs, sh.d), sh.d ** -0.5, torch.bfloat16, DEV)
        w["sd"] = synth.normal(seed, 28, (ns, sh.d, ffs), ffs ** -0.5, torch.bfloat16, DEV)
    else:
        w["sg"] = w["su"] = w["sd"] = None
    return w


def _both_paths(sh, x, perm_token, offsets, w):
    """(y_perm, y_shared) of the two-step path and of the fused path."""
    cfg = moe.MoeConfig.of(sh)
    ws = moe.alloc_workspace(cfg)
    n = sh.T * sh.K
    ns = sh.n_shared
    x_perm = x[perm_token.long()].contiguous()
    out = []
    for fused in (False, True):
        y = torch.full((n, sh.d), float("nan"), dtype=torch.bfloat16, device=DEV)
        ysh = torch.full((sh.T, sh.d), float("nan"), dtype=torch.bfloat16, device=DEV) if ns else None
        if fused:
            moe.moe_expert_ffn_gather(cfg, x, perm_token, offsets, w["wg"], w["wu"], w["wd"], y,
                                      w["sg"], w["su"], w["sd"], ysh, ws)
        else:
            moe.moe_expert_ffn(cfg, x_perm, offsets, w["wg"], w["wu"], w["wd"], y,
                               x if ns else None, w["sg"], w["su"], w["sd"], ysh, ws)
        assert moe.moe_read_device_status(ws) == moe.MOE_OK
        out.append((y, ysh))
    return out


def _assert_bits_equal(a, b):
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("name", ["tiny", "ragged", "ragged2", "noshared", "mid"])
def test_fused_gather_is_bit_identical_on_real_routing(orc, name):
    sh = H.shape(name)
    inp = synth.make_inputs(sh, DEV, weights=False)
    cfg = moe.MoeConfig.of(sh)
    ws = moe.alloc_workspace(cfg)
    idx = torch.empty(sh.T, sh.K, dtype=torch.int32, device=DEV)
    wt = torch.empty(sh.T, sh.K, dtype=torch.float32, device=DEV)
    moe.moe_route(cfg, inp["x"], inp["router_w"], inp.get("logit_offset"), inp["bias"], idx, wt,
                  ws=ws)
    i32 = lambda *s: torch.empty(*s, dtype=torch.int32, device=DEV)  # noqa: E731
    counts, offsets, send, send_tok = i32(sh.E), i32(sh.E + 1), i32(sh.G, sh.G), i32(sh.G, sh.G)
    perm, inv = i32(sh.T * sh.K), i32(sh.T, sh.K)
    moe.moe_dispatch(cfg, inp["x"], idx, counts, offsets, send, send_tok, perm, inv, None, ws)
    w = _weights(sh, sh.seed)
    (y0, s0), (y1, s1) = _both_paths(sh, inp["x"], perm, offsets, w)
    _assert_bits_equal(y0, y1)
    if sh.n_shared:
        _assert_bits_equal(s0, s1)
    # the fused path against the oracle on a sample of rows
    n = sh.T * sh.K
    off_h = offsets.cpu().numpy()
    rows = np.unique(np.linspace(0, n - 1, min(n, 48)).astype(np.int64))
    expert_of = np.searchsorted(off_h, rows, side="right") - 1
    xh, ph = inp["x"].cpu(), perm.cpu().numpy()
    ref = np.stack([orc.ffn_row(xh[ph[r]], w["wg"][e].cpu(), w["wu"][e].cpu(), w["wd"][e].cpu())
                    for r, e in zip(rows, expert_of)])
    frob, elem = H.compare_out(y1[torch.as_tensor(rows, device=DEV)], ref)
    assert frob <= H.TOL_FROB and elem <= H.TOL_ELEM, (frob, elem)


def test_fused_gather_segment_edges_and_repeated_rows():
    """Segments of 0, 1, 127, 128, 129, 255, 256, 257 rows; gathered token
    rows repeat and come in any order."""
    counts = [0, 1, 127, 128, 129, 255, 256, 257, 0, 999]
    T = 64                                           # distinct rows behind x
    n = sum(counts)
    sh = synth.MoeShape("edges", T=n, d=192, E=len(counts), G=1, K=1, M=1, d_ff=192,
                        n_shared=1, d_ff_shared=192, x_sigma=1, e_sigma=1, bias_sigma=0)
    base = synth.normal(3, 31, (T, sh.d), 1.0, torch.bfloat16, DEV)
    perm = (synth.uniform01(3, 32, (n,), DEV) * T).long().clamp(max=T - 1)
    x = base[perm].contiguous()                       # x has n rows (many equal)
    perm_token = torch.randperm(n, generator=torch.Generator().manual_seed(4)).to(DEV).to(torch.int32)
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32, device=DEV)
    w = _weights(sh, 5)
    (y0, s0), (y1, s1) = _both_paths(sh, x, perm_token, offsets, w)
    _assert_bits_equal(y0, y1)
    _assert_bits_equal(s0, s1)


def test_fused_gather_v3_bit_identical():
    sh = H.shape("v3")
    inp = synth.make_inputs(sh, DEV)
    cfg = moe.MoeConfig.of(sh)
    ws = moe.alloc_workspace(cfg)
    o = moe.forward_outputs(cfg)
    moe.moe_forward(cfg, inp["x"], inp["router_w"], None, inp["bias"], inp["w_gate"], inp["w_up"],
                    inp["w_down"], inp["ws_gate"], inp["ws_up"], inp["ws_down"], o["out"],
                    o["topk_idx"], o["topk_w"], o["counts"], o["offsets"], ws=ws)
    perm = torch.empty(sh.T * sh.K, dtype=torch.int32, device=DEV)
    inv = torch.empty(sh.T, sh.K, dtype=torch.int32, device=DEV)
    moe.moe_dispatch(cfg, inp["x"], o["topk_idx"], o["counts"], o["offsets"], o["send"],
                     o["send_tok"], perm, inv, None, ws)
    w = {"wg": inp["w_gate"], "wu": inp["w_up"], "wd": inp["w_down"], "sg": inp["ws_gate"],
         "su": inp["ws_up"], "sd": inp["ws_down"]}
    (y0, s0), (y1, s1) = _both_paths(sh, inp["x"], perm, o["offsets"], w)
    _assert_bits_equal(y0, y1)
    _assert_bits_equal(s0, s1)
    # moe_forward (fused) equals the staged two-step path end to end
    out2 = torch.empty_like(o["out"])
    moe.moe_combine(cfg, y0, inv, o["topk_w"], s0, out2)
    _assert_bits_equal(o["out"], out2)


def test_fused_gather_flags_bad_token_ids():
    sh = H.RAGGED2.replace(T=64, n_shared=0, d_ff_shared=0)
    cfg = moe.MoeConfig.of(sh)
    n = sh.T * sh.K
    x = synth.normal(1, 21, (sh.T, sh.d), 1.0, torch.bfloat16, DEV)
    w = _weights(sh, 1)
    offsets = torch.linspace(0, n, sh.E + 1, device=DEV).to(torch.int32)
    perm = (torch.arange(n, device=DEV) % sh.T).to(torch.int32)
    perm[5] = sh.T          # one past the last row of x
    perm[77] = -3
    y = torch.zeros(n, sh.d, dtype=torch.bfloat16, device=DEV)
    ws = moe.alloc_workspace(cfg)
    moe.moe_expert_ffn_gather(cfg, x, perm, offsets, w["wg"], w["wu"], w["wd"], y, None, None,
                              None, None, ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_DEVICE_FAULT
