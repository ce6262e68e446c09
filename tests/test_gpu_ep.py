"""Expert parallelism, emulated: every rank of one EP step on this GPU, with
the EP kernels (plan, dispatch with stores through the pointer table, expert
FFN of the rank's experts, combine with loads through the table).

Bars: the plan bit-exact against the oracle's row placement; with the batch
split into equal contiguous chunks the layer's routing, counts and output
equal moe_forward's bit for bit (every row meets the same arithmetic) where
the router reduces d in one range on both sides (d < 512); at the V3 sizes
the output is within the layer's bars of the oracle.
"""
import gc
import math

import numpy as np
import pytest
import torch

import synth
from tests import harness as H

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import combine_expert_ffn_b200 as moe
    from combine_expert_ffn_b200 import ep
else:  # collected on CPU-only machines, skipped by the marker filter
    moe = ep = None

DEV = "cuda"


@pytest.fixture(autouse=True)
def _free_gpu():
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _forward(sh, inp, router=None, token_ids=None, payload=None):
    cfg = moe.MoeConfig.of(sh, router=router, payload=payload)
    ws = moe.alloc_workspace(cfg)
    o = moe.forward_outputs(cfg)
    moe.moe_forward(cfg, inp["x"], inp["router_w"], inp.get("logit_offset"), inp["bias"],
                    inp["w_gate"], inp["w_up"], inp["w_down"], inp.get("ws_gate"),
                    inp.get("ws_up"), inp.get("ws_down"), o["out"], o["topk_idx"], o["topk_w"],
                    o["counts"], offsets=o["offsets"], ws=ws, token_ids=token_ids)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    return o


CASES = [("ragged", 2, 0), ("noshared", 2, 0), ("noshared", 4, 0), ("ragged2", 5, 0),
         ("ragged", 2, 2), ("noshared", 4, 1)]


@pytest.mark.parametrize("name,world,router", CASES)
def test_emulated_ep_equals_single_gpu_forward(orc, name, world, router):
    sh = H.shape(name)
    inp = synth.make_inputs(sh, DEV)
    ids = synth.token_ids(sh.seed, sh.T, device=DEV) if router == 2 else None
    ref = _forward(sh, inp, router, ids)
    out, ranks = ep.emulate_forward(sh, inp, world, router=router, token_ids=ids)
    torch.cuda.synchronize()
    for st in ranks:
        assert int(st.status.item()) == moe.MOE_OK
        assert moe.moe_read_device_status(st.ws) == moe.MOE_OK
    assert torch.equal(torch.cat([st.topk_idx for st in ranks]), ref["topk_idx"])
    assert torch.equal(torch.cat([st.topk_w for st in ranks]), ref["topk_w"])
    assert torch.equal(sum(st.counts for st in ranks), ref["counts"])
    assert torch.equal(out.view(torch.int16), ref["out"].view(torch.int16))
    # the plan kernel against the oracle's row placement
    counts_all = torch.stack([st.counts for st in ranks]).cpu().numpy()
    base, loff = orc.ep_plan(counts_all)
    for r, st in enumerate(ranks):
        np.testing.assert_array_equal(st.base.cpu().numpy(), base[r])
        np.testing.assert_array_equal(st.local_offsets.cpu().numpy(), loff[r])


def test_emulated_ep_v3_matches_oracle(orc):
    sh = H.shape("v3")
    inp = synth.make_inputs(sh, DEV)
    out, ranks = ep.emulate_forward(sh, inp, 8)
    torch.cuda.synchronize()
    for st in ranks:
        assert int(st.status.item()) == moe.MOE_OK
    rows = np.unique(np.linspace(0, sh.T - 1, 8).astype(np.int64))
    ref_out, ref_idx, _, ref_s = H.oracle_layer_sample(orc, sh, inp, rows)
    gi = torch.cat([st.topk_idx for st in ranks]).cpu().numpy()[rows]
    keep = [r for r in range(len(rows)) if np.array_equal(gi[r], ref_idx[r])]
    for r in set(range(len(rows))) - set(keep):
        assert H.near_tie_certified(sh, ref_s[r], inp["bias"].cpu().numpy(), gi[r], ref_idx[r])
    frob, elem = H.compare_out(out[torch.as_tensor(rows[keep], device=DEV)], ref_out[keep])
    assert frob <= H.TOL_FROB and elem <= H.TOL_ELEM, (frob, elem)


# d % 128 == 0 for the FP8 payload, one router range over d, shared experts
EP_FP8 = synth.MoeShape("ep_fp8", T=256, d=384, E=16, G=4, K=4, M=2, d_ff=192, n_shared=1,
                        d_ff_shared=128, x_sigma=1.0, e_sigma=1 / math.sqrt(384),
                        bias_sigma=0.1, seed=11)


@pytest.mark.parametrize("name,world", [("ep_fp8", 2), ("ep_fp8", 4), ("noshared", 2),
                                        ("noshared", 4)])
def test_emulated_ep_fp8_payload_equals_single_gpu(name, world):
    """The FP8 dispatch payload across ranks: the codes and scales every owner
    receives are the rows of the single-GPU FP8 dispatch of the whole batch
    restricted to its experts, and the layer's output equals moe_forward's
    with the FP8 payload bit for bit."""
    sh = EP_FP8 if name == "ep_fp8" else H.shape(name)
    inp = synth.make_inputs(sh, DEV)
    fp8 = moe.MOE_PAYLOAD_FP8
    ref = _forward(sh, inp, payload=fp8)
    out, ranks = ep.emulate_forward(sh, inp, world, payload=fp8)
    torch.cuda.synchronize()
    for st in ranks:
        assert int(st.status.item()) == moe.MOE_OK
        assert moe.moe_read_device_status(st.ws) == moe.MOE_OK
    assert torch.equal(torch.cat([st.topk_idx for st in ranks]), ref["topk_idx"])
    assert torch.equal(out.view(torch.int16), ref["out"].view(torch.int16))
    # the single-GPU FP8 dispatch of the whole batch
    cfg8 = moe.MoeConfig.of(sh, payload=fp8)
    ws = moe.alloc_workspace(cfg8)
    T, K, E, G = sh.T, sh.K, sh.E, sh.G
    i32 = dict(dtype=torch.int32, device=DEV)
    counts, offsets = torch.empty(E, **i32), torch.empty(E + 1, **i32)
    send, send_tok = torch.empty(G, G, **i32), torch.empty(G, G, **i32)
    perm, inv = torch.empty(T * K, **i32), torch.empty(T, K, **i32)
    xq = torch.empty(T * K, sh.d, dtype=torch.uint8, device=DEV)
    xs = torch.empty(T * K, sh.d // 128, dtype=torch.float32, device=DEV)
    moe.moe_dispatch_fp8(cfg8, inp["x"], ref["topk_idx"], counts, offsets, send, send_tok, perm,
                         inv, xq, xs, ws)
    torch.cuda.synchronize()
    El = E // world
    off = offsets.cpu().numpy()
    for o, st in enumerate(ranks):
        lo, hi = int(off[o * El]), int(off[(o + 1) * El])
        n = int(st.local_offsets[El].item())
        assert n == hi - lo
        assert torch.equal(st.recv_q[:n], xq[lo:hi])
        assert torch.equal(st.recv_scale[:n].view(torch.int32), xs[lo:hi].view(torch.int32))


def test_emulated_ep_fp8_v3_matches_oracle(orc):
    sh = H.shape("v3")
    inp = synth.make_inputs(sh, DEV)
    out, ranks = ep.emulate_forward(sh, inp, 8, payload=moe.MOE_PAYLOAD_FP8)
    torch.cuda.synchronize()
    for st in ranks:
        assert int(st.status.item()) == moe.MOE_OK
    rows = np.unique(np.linspace(0, sh.T - 1, 6).astype(np.int64))
    ref_out, ref_idx, _, ref_s = H.oracle_layer_sample(orc, sh, inp, rows, payload=1)
    gi = torch.cat([st.topk_idx for st in ranks]).cpu().numpy()[rows]
    keep = [r for r in range(len(rows)) if np.array_equal(gi[r], ref_idx[r])]
    for r in set(range(len(rows))) - set(keep):
        assert H.near_tie_certified(sh, ref_s[r], inp["bias"].cpu().numpy(), gi[r], ref_idx[r])
    frob, elem = H.compare_out(out[torch.as_tensor(rows[keep], device=DEV)], ref_out[keep])
    assert frob <= H.TOL_FROB and elem <= H.TOL_ELEM, (frob, elem)


def test_emulated_ep_owner_with_no_rows():
    """A bias that keeps every token out of rank 1's experts (groups 2 and 3
    of 4): rank 1 receives no rows, runs only its shared experts, and the
    layer still equals moe_forward bit for bit."""
    sh = H.shape("ragged")                       # E 12, G 4, M 2: rank 1 owns groups 2, 3
    inp = synth.make_inputs(sh, DEV)
    bias = inp["bias"].clone()
    bias[sh.E // 2:] = -10.0
    inp = dict(inp, bias=bias)
    ref = _forward(sh, inp)
    assert int(ref["counts"][sh.E // 2:].sum()) == 0
    out, ranks = ep.emulate_forward(sh, inp, 2)
    torch.cuda.synchronize()
    assert int(ranks[1].local_offsets[-1].item()) == 0
    for st in ranks:
        assert int(st.status.item()) == moe.MOE_OK
        assert moe.moe_read_device_status(st.ws) == moe.MOE_OK
    assert torch.equal(out.view(torch.int16), ref["out"].view(torch.int16))


def test_emulated_ep_world_one_is_the_single_gpu_layer():
    sh = H.shape("ragged")
    inp = synth.make_inputs(sh, DEV)
    ref = _forward(sh, inp)
    out, ranks = ep.emulate_forward(sh, inp, 1)
    torch.cuda.synchronize()
    assert int(ranks[0].status.item()) == moe.MOE_OK
    assert torch.equal(out.view(torch.int16), ref["out"].view(torch.int16))
    assert torch.equal(ranks[0].local_offsets, ref["offsets"])


def test_emulated_ep_empty_batch():
    sh = H.shape("ragged")
    inp = synth.make_inputs(sh, DEV)
    empty = sh.replace(T=0)
    inp = dict(inp, x=inp["x"][:0])
    out, ranks = ep.emulate_forward(empty, inp, 2)
    torch.cuda.synchronize()
    assert out.shape == (0, sh.d)
    for st in ranks:
        assert int(st.status.item()) == moe.MOE_OK
        assert int(st.local_offsets[-1].item()) == 0


def test_emulated_ep_maximum_world(orc):
    """64 ranks (the largest world) of one expert each on the mid workload
    (T=4096, d=2048, E=64, K=6): sampled tokens within the layer's bars of the
    oracle."""
    sh = H.shape("mid")
    inp = synth.make_inputs(sh, DEV)
    out, ranks = ep.emulate_forward(sh, inp, 64)
    torch.cuda.synchronize()
    for st in ranks:
        assert int(st.status.item()) == moe.MOE_OK
    counts_all = torch.stack([st.counts for st in ranks]).cpu().numpy()
    base, loff = orc.ep_plan(counts_all)
    for r, st in enumerate(ranks):
        np.testing.assert_array_equal(st.base.cpu().numpy(), base[r])
        np.testing.assert_array_equal(st.local_offsets.cpu().numpy(), loff[r])
    rows = np.unique(np.linspace(0, sh.T - 1, 8).astype(np.int64))
    ref_out, ref_idx, _, ref_s = H.oracle_layer_sample(orc, sh, inp, rows)
    gi = torch.cat([st.topk_idx for st in ranks]).cpu().numpy()[rows]
    keep = [r for r in range(len(rows)) if np.array_equal(gi[r], ref_idx[r])]
    for r in set(range(len(rows))) - set(keep):
        assert H.near_tie_certified(sh, ref_s[r], inp["bias"].cpu().numpy(), gi[r], ref_idx[r])
    frob, elem = H.compare_out(out[torch.as_tensor(rows[keep], device=DEV)], ref_out[keep])
    assert frob <= H.TOL_FROB and elem <= H.TOL_ELEM, (frob, elem)


@pytest.mark.parametrize("name,world", [("ragged", 2), ("noshared", 4), ("ragged2", 5),
                                        ("ragged", 3)])
def test_emulated_ep_dedup_dispatch(orc, name, world):
    """One row per (token, owner) and a fan-out index per copy: the token
    plans and bases equal the oracle's bit for bit, every owner's fanned-out
    rows equal what the per-copy dispatch stores, and the layer equals
    moe_forward bit for bit."""
    sh = H.shape(name)
    inp = synth.make_inputs(sh, DEV)
    ref = _forward(sh, inp)
    out, ranks = ep.emulate_forward(sh, inp, world, dedup=True)
    _, plain = ep.emulate_forward(sh, inp, world)
    torch.cuda.synchronize()
    for st in ranks:
        assert int(st.status.item()) == moe.MOE_OK
        assert moe.moe_read_device_status(st.ws) == moe.MOE_OK
    assert torch.equal(out.view(torch.int16), ref["out"].view(torch.int16))
    plans = [orc.ep_token_plan(st.topk_idx.cpu().numpy(), sh.E, world) for st in ranks]
    tok_counts_all = np.stack([p[1] for p in plans])
    tok_base = orc.ep_token_base(tok_counts_all)
    El = sh.E // world
    for r, st in enumerate(ranks):
        np.testing.assert_array_equal(st.tok_slot.cpu().numpy(), plans[r][0])
        np.testing.assert_array_equal(st.tok_counts.cpu().numpy(), plans[r][1])
        np.testing.assert_array_equal(st.tok_base[:world].cpu().numpy(), tok_base[r])
        assert int(st.tok_base[world].item()) == int(tok_counts_all[:, r].sum())
        n = int(st.local_offsets[El].item())
        assert torch.equal(st.recv_x[:n].view(torch.int16), plain[r].recv_x[:n].view(torch.int16))



@pytest.mark.parametrize("name,world", [("ragged", 2), ("ragged", 3), ("noshared", 4),
                                        ("ragged2", 5)])
def test_emulated_ep_dedup_combine(orc, name, world):
    """Both exchanges at (token, owner) granularity: each owner sums its
    copies of a token into one bf16 partial row.  One more bf16 rounding than
    the single-GPU combine, so: every token within the layer's bars of the
    oracle, and close to the per-copy EP path."""
    sh = H.shape(name)
    inp = synth.make_inputs(sh, DEV)
    out, ranks = ep.emulate_forward(sh, inp, world, dedup=True, dedup_combine=True)
    plain, _ = ep.emulate_forward(sh, inp, world)
    torch.cuda.synchronize()
    for st in ranks:
        assert int(st.status.item()) == moe.MOE_OK
        assert moe.moe_read_device_status(st.ws) == moe.MOE_OK
    rows = np.arange(sh.T)
    ref_out, ref_idx, _, ref_s = H.oracle_layer_sample(orc, sh, inp, rows)
    gi = torch.cat([st.topk_idx for st in ranks]).cpu().numpy()
    keep = [r for r in rows if np.array_equal(gi[r], ref_idx[r])]
    for r in set(rows.tolist()) - set(keep):
        assert H.near_tie_certified(sh, ref_s[r], inp["bias"].cpu().numpy(), gi[r], ref_idx[r])
    frob, elem = H.compare_out(out[torch.as_tensor(keep, device=DEV)], ref_out[keep])
    assert frob <= H.TOL_FROB and elem <= H.TOL_ELEM, (frob, elem)
    a, b = out.float(), plain.float()
    assert float((a - b).norm() / b.norm()) <= H.TOL_FROB


@pytest.mark.parametrize("name,world", [("ragged", 2), ("ragged", 3), ("noshared", 4),
                                        ("ragged2", 5)])
def test_dedup_dispatch_with_plan_equals_two_launches(name, world):
    """moe_ep_dispatch_dedup_plan (one launch) writes what moe_ep_dispatch_dedup
    followed by moe_ep_combine_plan write: token rows, fan-out indices and the
    combine's lists, gates and counts, bit for bit; the counts add up to the
    copies each owner received."""
    sh = H.shape(name)
    inp = synth.make_inputs(sh, DEV)
    ems = []
    for fused in (True, False):
        em = ep.EmulatedEP(sh, inp, world, dedup=True, dedup_combine=True)
        for st in em.ranks:
            st.fused_plan = fused
        em.forward()
        ems.append(em)
    torch.cuda.synchronize()
    K, El = sh.K, sh.E // world
    for sa, sb in zip(ems[0].ranks, ems[1].ranks):
        for st in (sa, sb):
            assert int(st.status.item()) == moe.MOE_OK
            assert moe.moe_read_device_status(st.ws) == moe.MOE_OK
        n = int(sa.tok_base[world].item())
        m = int(sa.local_offsets[El].item())
        assert n == int(sb.tok_base[world].item()) and m == int(sb.local_offsets[El].item())
        assert torch.equal(sa.recv_tok[:n].view(torch.int16), sb.recv_tok[:n].view(torch.int16))
        assert torch.equal(sa.recv_idx[:m], sb.recv_idx[:m])
        cnt = sa.recv_lcnt[:n]
        assert torch.equal(cnt, sb.recv_lcnt[:n])
        assert bool(((cnt >= 1) & (cnt <= K)).all()) and int(cnt.sum()) == m
        used = (torch.arange(K, device=DEV)[None, :] < cnt[:, None].long()).reshape(-1)
        assert torch.equal(sa.recv_list[:n * K][used], sb.recv_list[:n * K][used])
        assert torch.equal(sa.recv_lw[:n * K][used].view(torch.int32),
                           sb.recv_lw[:n * K][used].view(torch.int32))
        assert torch.equal(sa.out.view(torch.int16), sb.out.view(torch.int16))


def test_emulated_ep_dedup_combine_v3_matches_oracle(orc):
    sh = H.shape("v3")
    inp = synth.make_inputs(sh, DEV)
    out, ranks = ep.emulate_forward(sh, inp, 8, dedup=True, dedup_combine=True)
    torch.cuda.synchronize()
    for st in ranks:
        assert int(st.status.item()) == moe.MOE_OK
    rows = np.unique(np.linspace(0, sh.T - 1, 6).astype(np.int64))
    ref_out, ref_idx, _, ref_s = H.oracle_layer_sample(orc, sh, inp, rows)
    gi = torch.cat([st.topk_idx for st in ranks]).cpu().numpy()[rows]
    keep = [r for r in range(len(rows)) if np.array_equal(gi[r], ref_idx[r])]
    for r in set(range(len(rows))) - set(keep):
        assert H.near_tie_certified(sh, ref_s[r], inp["bias"].cpu().numpy(), gi[r], ref_idx[r])
    frob, elem = H.compare_out(out[torch.as_tensor(rows[keep], device=DEV)], ref_out[keep])
    assert frob <= H.TOL_FROB and elem <= H.TOL_ELEM, (frob, elem)


@pytest.mark.parametrize("name,world", [("ep_fp8", 2), ("ep_fp8", 4), ("noshared", 4)])
def test_emulated_ep_dedup_fp8_payload(name, world):
    """The FP8 payload sent once per (token, owner): every owner's fanned-out
    codes and scales equal what the per-copy FP8 dispatch stores, and the
    layer equals moe_forward with the FP8 payload bit for bit."""
    sh = EP_FP8 if name == "ep_fp8" else H.shape(name)
    inp = synth.make_inputs(sh, DEV)
    fp8 = moe.MOE_PAYLOAD_FP8
    ref = _forward(sh, inp, payload=fp8)
    out, ranks = ep.emulate_forward(sh, inp, world, payload=fp8, dedup=True)
    _, plain = ep.emulate_forward(sh, inp, world, payload=fp8)
    torch.cuda.synchronize()
    for st in ranks:
        assert int(st.status.item()) == moe.MOE_OK
        assert moe.moe_read_device_status(st.ws) == moe.MOE_OK
    assert torch.equal(out.view(torch.int16), ref["out"].view(torch.int16))
    El = sh.E // world
    for r, st in enumerate(ranks):
        n = int(st.local_offsets[El].item())
        assert torch.equal(st.recv_q[:n], plain[r].recv_q[:n])
        assert torch.equal(st.recv_scale[:n].view(torch.int32),
                           plain[r].recv_scale[:n].view(torch.int32))


def test_emulated_ep_world_one_maximum_experts():
    """One rank owning all 1024 experts (the largest E): the last local segment's
    end (local_offsets[1024], one past the plan kernel's last thread) is written,
    and the layer equals moe_forward bit for bit."""
    sh = synth.MoeShape("ep_max_experts", T=512, d=128, E=1024, G=64, K=32, M=16, d_ff=64,
                        n_shared=1, d_ff_shared=64, x_sigma=1.0, e_sigma=1 / math.sqrt(128),
                        bias_sigma=0.1, seed=11)
    inp = synth.make_inputs(sh, DEV)
    ref = _forward(sh, inp)
    out, ranks = ep.emulate_forward(sh, inp, 1)
    torch.cuda.synchronize()
    assert int(ranks[0].status.item()) == moe.MOE_OK
    assert torch.equal(ranks[0].local_offsets, ref["offsets"])
    assert int(ranks[0].local_offsets[-1].item()) == sh.T * sh.K
    assert torch.equal(out.view(torch.int16), ref["out"].view(torch.int16))
