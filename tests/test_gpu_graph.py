"""moe_forward inside a CUDA graph.

The forward only enqueues kernels on the caller's stream (no allocation, no
synchronisation, no host read-back), so it can be captured once and replayed:
the replay must give the eager forward's bits, also after the input buffer is
refilled with another batch.  With row-major and with tile-packed weights.
"""
import gc

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


@pytest.mark.parametrize("name,router,payload,packed", [
    ("tiny", 0, 0, False), ("ragged2", 1, 0, False), ("noshared", 0, 1, False),
    ("mid", 2, 0, False),
    # the tile-packed weights; ragged at 2048 tokens averages 683 rows per expert, so
    # its GEMMs are the paired-row-tile kernels whose tile counters a memset resets
    ("tiny", 0, 0, True), ("mid", 0, 0, True), ("ragged_2048", 0, 0, True)])
def test_forward_replays_from_a_cuda_graph(name, router, payload, packed):
    sh = H.RAGGED.replace(name=name, T=2048) if name == "ragged_2048" else H.shape(name)
    inp = synth.make_inputs(sh, DEV)
    cfg = moe.MoeConfig.of(sh, router=router, payload=payload)
    ws = moe.alloc_workspace(cfg)
    o = moe.forward_outputs(cfg)
    ids = synth.token_ids(sh.seed, sh.T, device=DEV)
    x = inp["x"].clone()
    pw = moe.pack_weights(cfg, inp["w_gate"], inp["w_up"], inp["w_down"], inp.get("ws_gate"),
                          inp.get("ws_up"), inp.get("ws_down")) if packed else None

    def forward(stream=None):
        if packed:
            moe.moe_forward_packed(cfg, x, inp["router_w"], inp.get("logit_offset"), inp["bias"],
                                   pw, o["out"], o["topk_idx"], o["topk_w"], o["counts"],
                                   o["offsets"], o["send"], o["send_tok"], ws=ws, stream=stream,
                                   token_ids=ids)
            return
        moe.moe_forward(cfg, x, inp["router_w"], inp.get("logit_offset"), inp["bias"],
                        inp["w_gate"], inp["w_up"], inp["w_down"], inp.get("ws_gate"),
                        inp.get("ws_up"), inp.get("ws_down"), o["out"], o["topk_idx"],
                        o["topk_w"], o["counts"], o["offsets"], o["send"], o["send_tok"], ws=ws,
                        stream=stream, token_ids=ids)

    forward()                                     # first call outside the capture
    torch.cuda.synchronize()
    eager = {k: v.clone() for k, v in o.items()}
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            forward(stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for v in o.values():
        v.zero_()
    g.replay()
    torch.cuda.synchronize()
    for k in eager:
        assert torch.equal(o[k], eager[k]), k
    # another batch in the same buffer: the replay equals an eager forward of it
    x.copy_(synth.normal(sh.seed + 1, synth.TENSOR_IDS["x"], (sh.T, sh.d), sh.x_sigma,
                         torch.bfloat16, DEV))
    g.replay()
    torch.cuda.synchronize()
    replayed = {k: v.clone() for k, v in o.items()}
    forward()
    torch.cuda.synchronize()
    for k in replayed:
        assert torch.equal(o[k], replayed[k]), k
    assert moe.moe_read_device_status(ws) == moe.MOE_OK
    del g
