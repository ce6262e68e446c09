"""The multi-process expert-parallel layer (EPLayer) with its ranks as
separate processes sharing one GPU: every rank maps the others' receive
buffers by CUDA IPC (same device, different processes), the kernels store
and load through those mappings, and the collectives are gloo with the
step's stream synchronised before each (none of the EP kernels waits on
another rank, so the ranks never need to run at the same time).

Bar: two consecutive steps (the buffers are reused) both equal moe_forward on
the whole batch bit for bit; no status word is set.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, name, payload, dedup, q, dedup_combine=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import synth
        from tests import harness as H
        import combine_expert_ffn_b200 as moe
        from combine_expert_ffn_b200.ep import EPLayer
        sh = H.shape(name)
        inp = synth.make_inputs(sh, "cuda")
        Tr, El = sh.T // world, sh.E // world
        sl = slice(rank * El, (rank + 1) * El)
        layer = EPLayer(sh.replace(T=Tr), None, inp["router_w"], inp["bias"], inp["w_gate"][sl],
                        inp["w_up"][sl], inp["w_down"][sl], inp.get("ws_gate"), inp.get("ws_up"),
                        inp.get("ws_down"), logit_offset=inp.get("logit_offset"), payload=payload,
                        dedup=dedup, dedup_combine=dedup_combine)
        x = inp["x"][rank * Tr:(rank + 1) * Tr]
        outs = []
        for _ in range(2):
            out = layer.forward(x)
            torch.cuda.synchronize()
            outs.append(out.cpu().view(torch.int16).numpy().copy())
        status = int(layer.st.status.item())
        dstatus = moe.moe_read_device_status(layer.st.ws)
        layer.close()
        q.put((rank, outs, status, dstatus, None))
    except Exception as e:  # reported to the parent, then re-raised
        q.put((rank, None, None, None, repr(e)))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,world,payload,dedup,dedup_combine",
                         [("ragged", 2, 0, False, False), ("ragged", 3, 0, False, False),
                          ("noshared", 2, 1, False, False), ("ragged", 3, 0, True, False),
                          ("ragged", 3, 0, True, True), ("noshared", 2, 1, True, False)])
def test_ep_layer_processes_on_one_gpu_equal_single_gpu_forward(name, world, payload, dedup,
                                                                dedup_combine):
    """Bit for bit except with the deduplicated combine (one more bf16
    rounding of each owner's partial sum): there, within the layer's bars of
    the single-GPU output, and the two steps equal each other."""
    import synth
    from tests import harness as H
    import combine_expert_ffn_b200 as moe
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main,
                         args=(r, world, port, name, payload, dedup, q, dedup_combine))
             for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):
            rank, outs, status, dstatus, err = q.get(timeout=300)
            assert err is None, f"rank {rank}: {err}"
            got[rank] = (outs, status, dstatus)
    finally:
        for p in procs:
            p.join(timeout=120)
            if p.is_alive():
                p.kill()
    for p in procs:
        assert p.exitcode == 0
    sh = H.shape(name)
    inp = synth.make_inputs(sh, "cuda")
    cfg = moe.MoeConfig.of(sh, payload=payload)
    ws = moe.alloc_workspace(cfg)
    o = moe.forward_outputs(cfg)
    moe.moe_forward(cfg, inp["x"], inp["router_w"], inp.get("logit_offset"), inp["bias"],
                    inp["w_gate"], inp["w_up"], inp["w_down"], inp.get("ws_gate"),
                    inp.get("ws_up"), inp.get("ws_down"), o["out"], ws=ws)
    ref = o["out"].cpu().view(torch.int16).numpy()
    Tr = sh.T // world
    for r in range(world):
        outs, status, dstatus = got[r]
        assert status == moe.MOE_OK and dstatus == moe.MOE_OK
        np.testing.assert_array_equal(outs[0], outs[1])
        mine = ref[r * Tr:(r + 1) * Tr]
        if not dedup_combine:
            np.testing.assert_array_equal(outs[0], mine)
        else:
            a = torch.from_numpy(outs[0]).view(torch.bfloat16).float()
            b = torch.from_numpy(mine.copy()).view(torch.bfloat16).float()
            assert float((a - b).norm() / b.norm()) <= H.TOL_FROB
