"""moe_dispatch_noalloc: the dispatch for callers that cannot allocate device memory.

A serving runtime that owns the whole HBM budget through its own pool, or a
latency-critical path that cannot afford cudaMalloc's implicit device
synchronisation, cannot hand the library a workspace.  The no-allocation
entry point keeps the dispatch scratch in a fixed static device array
instead; these tests check, through the C ABI, that it gives exactly what
moe_dispatch gives (integer outputs: bit for bit) on two calls in a row that
share that array, and that sizes beyond the array are refused up front.
This file is collected last so that a failure here never hides another test.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import synth
from tests import harness as H

SCRATCH_BYTES = 4 << 20


def _scratch_need(T, E, G):
    nblk = (T + 255) // 256
    r = lambda v: (v + 255) // 256 * 256
    return 256 + 2 * r(4 * E * nblk) + 2 * r(4 * nblk * G * G)


def test_sizes_beyond_the_static_scratch_are_refused():
    # 4 MiB holds every named workload; E = 1024 experts, G = 64 groups and
    # T = 131072 tokens does not.  Refused before any CUDA call.
    import os
    import importlib.util
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("_moe_build", os.path.join(root, "combine_expert_ffn_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    import combine_expert_ffn_b200 as moe
    for name in ("tiny", "mid", "v3", "decode", "skew"):
        sh = synth.config(name)
        assert _scratch_need(sh.T, sh.E, sh.G) <= SCRATCH_BYTES
    big = moe.MoeConfig(T=131072, d=128, E=1024, G=64, K=8, M=4, d_ff=64, n_shared=0, d_ff_shared=0)
    assert _scratch_need(big.T, big.E, big.G) > SCRATCH_BYTES
    fake = C.c_void_p(1 << 20)
    st = moe._lib.moe_dispatch_noalloc(C.byref(big), fake, fake, fake, fake, fake, fake, fake, fake,
                                       None, None, None)
    assert st == moe.MOE_ERR_WORKSPACE_TOO_SMALL


def _outputs(sh, dev):
    i32 = lambda *s: torch.full(s, -7, dtype=torch.int32, device=dev)
    return {"counts": i32(sh.E), "offsets": i32(sh.E + 1), "send": i32(sh.G, sh.G),
            "send_tok": i32(sh.G, sh.G), "perm_token": i32(sh.T * sh.K), "inv_perm": i32(sh.T, sh.K),
            "x_perm": torch.zeros(sh.T * sh.K, sh.d, dtype=torch.bfloat16, device=dev)}


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["ragged2", "v3"])
def test_noalloc_dispatch_matches_workspace_dispatch_twice(name):
    import combine_expert_ffn_b200 as moe
    dev = "cuda"
    sh = H.shape(name)
    cfg = moe.MoeConfig.of(sh)
    ws = moe.alloc_workspace(cfg, dev)
    x = synth.normal(sh.seed, synth.TENSOR_IDS["x"], (sh.T, sh.d), 1.0, torch.bfloat16, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    # two calls in a row on different routings (balanced, then skewed): the
    # second reuses the static scratch the first one left behind
    for call, zipf in enumerate((0.0, 1.2)):
        topk = synth.random_routing(sh.seed + call, sh.T, sh.E, sh.K, zipf, dev)
        ref, got = _outputs(sh, dev), _outputs(sh, dev)
        moe.moe_dispatch(cfg, x, topk, ref["counts"], ref["offsets"], ref["send"], ref["send_tok"],
                         ref["perm_token"], ref["inv_perm"], ref["x_perm"], ws)
        moe.moe_dispatch_noalloc(cfg, x, topk, got["counts"], got["offsets"], got["send"],
                                 got["send_tok"], got["perm_token"], got["inv_perm"], got["x_perm"],
                                 device_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == moe.MOE_OK
        for k in ref:
            a, b = ref[k], got[k]
            if a.dtype == torch.bfloat16:
                a, b = a.view(torch.int16), b.view(torch.int16)
            assert torch.equal(a, b), (call, k)
        assert int(got["counts"].sum()) == sh.T * sh.K


@pytest.mark.gpu
def test_noalloc_dispatch_reports_bad_ids():
    import combine_expert_ffn_b200 as moe
    dev = "cuda"
    sh = H.RAGGED.replace(T=8, G=4)
    cfg = moe.MoeConfig.of(sh)
    x = synth.normal(1, 1, (sh.T, sh.d), 1.0, torch.bfloat16, dev)
    topk = torch.tensor([[0, 1, 2, 3]] * 8, dtype=torch.int32, device=dev)
    topk[5, 1] = -3
    o = _outputs(sh, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    moe.moe_dispatch_noalloc(cfg, x, topk, o["counts"], o["offsets"], o["send"], o["send_tok"],
                             o["perm_token"], o["inv_perm"], o["x_perm"], device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == moe.MOE_ERR_DEVICE_FAULT
