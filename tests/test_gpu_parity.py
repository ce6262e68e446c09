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
    moe.moe_clear_device_status(ws)
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
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
