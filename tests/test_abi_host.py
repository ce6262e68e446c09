"""Host-side checks of the C ABI that need no GPU.

The library must load and export every entry point ``include/moe.h``
declares, and validate its arguments before touching CUDA.  No call here
reaches a kernel launch: each one is rejected by validation first.
"""
import ctypes as C
import os
import re

import pytest
import torch

import synth
from tests import harness as H

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def moe():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_moe_build", os.path.join(ROOT, "combine_expert_ffn_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    import combine_expert_ffn_b200 as m
    return m


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"MOE_API[^;(]*?\b(moe_\w+)\(", text, flags=re.S)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for s in ("moe_route", "moe_route_select", "moe_dispatch", "moe_expert_ffn", "moe_combine",
              "moe_forward", "moe_workspace_size"):
        assert s in syms


def test_library_exports_every_declared_symbol(moe):
    lib = C.CDLL(moe.LIB_PATH)
    for s in declared_symbols():
        assert hasattr(lib, s), s
    assert sorted(moe.EXPORTS) == declared_symbols()


@pytest.mark.parametrize("name", list(H.SHAPES))
def test_known_workloads_are_supported(moe, name):
    cfg = moe.MoeConfig.of(H.shape(name))
    assert moe.moe_check_config(cfg) == moe.MOE_OK
    assert moe.moe_workspace_size(cfg) > 0


BAD = [
    dict(E=15),                    # E % G
    dict(K=3),                     # K % M
    dict(M=8),                     # M > G
    dict(K=32, M=2),               # K/M > E/G
    dict(d=100),                   # d % 64
    dict(d_ff=96),                 # d_ff % 64
    dict(d_ff_shared=32),          # d_ff_shared % 64
    dict(T=63),                    # T % G
    dict(E=2048, G=4),             # E > 1024
    dict(K=64, M=2, E=64, G=2),    # K > 32
    dict(T=-4),
    dict(d=0),
]


@pytest.mark.parametrize("kw", BAD)
def test_unsupported_shapes_are_rejected(moe, kw):
    cfg = moe.MoeConfig.of(synth.config("tiny").replace(**kw))
    assert moe.moe_check_config(cfg) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert moe.moe_workspace_size(cfg) == 0


def test_null_config(moe):
    assert moe._lib.moe_check_config(None) == moe.MOE_ERR_INVALID_ARG
    assert moe._lib.moe_workspace_size(None) == 0


def test_workspace_grows_with_tokens(moe):
    base = synth.config("v3")
    sizes = [moe.moe_workspace_size(moe.MoeConfig.of(base.replace(T=t))) for t in (0, 8, 64, 1024, 8192, 32768)]
    assert all(a <= b for a, b in zip(sizes, sizes[1:]))
    # the forward intermediates dominate: x_perm + y_perm + h + y_shared at least
    sh = base
    floor = 2 * sh.T * sh.K * sh.d * 2 + sh.T * sh.K * sh.d_ff * 2 + sh.T * sh.d * 2
    assert moe.moe_workspace_size(moe.MoeConfig.of(sh)) >= floor


def test_status_strings(moe):
    for code in range(8):
        assert moe.moe_status_string(code)
    assert moe.moe_status_string(99) == "unknown status"


def test_entry_points_validate_before_cuda(moe):
    cfg = moe.MoeConfig.of(synth.config("tiny"))
    ws_n = moe.moe_workspace_size(cfg)
    lib, fake = moe._lib, 1 << 20
    P = C.c_void_p
    # NULL required pointers
    assert lib.moe_route(C.byref(cfg), None, P(fake), None, None, P(fake), P(fake), P(fake),
                         None, 0, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_route_select(C.byref(cfg), None, None, P(fake), P(fake), None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(C.byref(cfg), None, P(fake), P(fake), None, P(fake), None) == moe.MOE_ERR_INVALID_ARG
    # misaligned buffer
    assert lib.moe_combine(C.byref(cfg), P(fake + 2), P(fake), P(fake), None, P(fake), None) == moe.MOE_ERR_INVALID_ARG
    # workspace too small
    args = [P(fake)] * 9
    assert lib.moe_dispatch(C.byref(cfg), *args, P(fake), ws_n - 1, None) == moe.MOE_ERR_WORKSPACE_TOO_SMALL
    assert lib.moe_forward(C.byref(cfg), *([P(fake)] * 18), P(fake), ws_n - 1, None) == moe.MOE_ERR_WORKSPACE_TOO_SMALL
    # misaligned workspace
    assert lib.moe_dispatch(C.byref(cfg), *args, P(fake + 16), ws_n, None) == moe.MOE_ERR_INVALID_ARG
    # unsupported shape wins over everything else
    bad = moe.MoeConfig.of(synth.config("tiny").replace(E=15))
    assert lib.moe_forward(C.byref(bad), *([None] * 18), None, 0, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    # self-test limits
    assert lib.moe_selftest_bounded_wait(10, P(fake), None) == moe.MOE_ERR_INVALID_ARG


def _packed_bytes(E, d, d_ff, n_shared, d_ff_shared):
    """The packed layout's size, restated from its definition in moe.h: 32 KB
    tiles of 256 weight rows x 64 k values; gate/up tiles hold 128 columns of
    h, down tiles 256 output columns."""
    up = lambda a, b: -(-a // b)  # noqa: E731
    ffs = n_shared * d_ff_shared
    tiles = E * up(d_ff, 128) * (d // 64) + E * up(d, 256) * (d_ff // 64)
    if ffs:
        tiles += up(ffs, 128) * (d // 64) + up(d, 256) * (ffs // 64)
    return tiles * 32768


@pytest.mark.parametrize("name", ["tiny", "ragged", "ragged2", "noshared", "mid", "v3"])
def test_packed_weights_size_and_validation(moe, name):
    sh = H.shape(name)
    cfg = moe.MoeConfig.of(sh)
    assert moe.moe_packed_weights_size(cfg) == _packed_bytes(sh.E, sh.d, sh.d_ff, sh.n_shared,
                                                             sh.d_ff_shared)
    assert moe.moe_packed_weights_size(moe.MoeConfig.of(sh.replace(E=sh.E + 1))) == 0
    lib, fake, P = moe._lib, 1 << 20, C.c_void_p
    c = C.byref(cfg)
    INV, UNS = moe.MOE_ERR_INVALID_ARG, moe.MOE_ERR_UNSUPPORTED_SHAPE
    w = [P(fake)] * 6                                  # w_gate .. ws_down
    assert lib.moe_pack_weights(c, *w, None, None) == INV               # packed
    bad = list(w)
    bad[1] = P(fake + 8)                               # misaligned w_up
    assert lib.moe_pack_weights(c, *bad, P(fake), None) == INV
    if sh.n_shared:
        bad = list(w)
        bad[3] = None                                  # ws_gate
        assert lib.moe_pack_weights(c, *bad, P(fake), None) == INV
    ws_n = moe.moe_workspace_size(cfg)
    # x_perm, offsets, packed, y_perm, x, y_shared
    f = [P(fake)] * 6
    assert lib.moe_expert_ffn_packed(c, *f, P(fake), ws_n - 1, None) == \
        moe.MOE_ERR_WORKSPACE_TOO_SMALL
    bad = list(f)
    bad[2] = None                                      # packed
    assert lib.moe_expert_ffn_packed(c, *bad, P(fake), ws_n, None) == INV
    assert lib.moe_expert_ffn_packed(c, *f, P(fake + 64), ws_n, None) == INV   # ws alignment
    # x, router_w, logit_offset, bias, token_ids, packed, out, then 6 optional outputs
    fw = [P(fake), P(fake), None, None, None, None, P(fake)] + [None] * 6
    assert lib.moe_forward_packed(c, *fw, P(fake), ws_n, None) == INV          # packed
    fw[5] = P(fake)
    fp8 = moe.MoeConfig.of(sh, payload=moe.MOE_PAYLOAD_FP8)
    if moe.moe_check_config(fp8) == moe.MOE_OK:
        assert lib.moe_forward_packed(C.byref(fp8), *fw, P(fake), ws_n, None) == UNS


def test_fused_gather_validates_before_cuda(moe):
    cfg = moe.MoeConfig.of(synth.config("tiny"))
    ws_n = moe.moe_workspace_size(cfg)
    lib, fake, P = moe._lib, 1 << 20, C.c_void_p
    args = [P(fake)] * 11                      # x .. y_shared
    assert lib.moe_expert_ffn_gather(C.byref(cfg), *args, P(fake), ws_n - 1, None) == \
        moe.MOE_ERR_WORKSPACE_TOO_SMALL
    bad = list(args)
    bad[1] = None                              # perm_token
    assert lib.moe_expert_ffn_gather(C.byref(cfg), *bad, P(fake), ws_n, None) == moe.MOE_ERR_INVALID_ARG
    bad = list(args)
    bad[0] = P(fake + 8)                       # misaligned x
    assert lib.moe_expert_ffn_gather(C.byref(cfg), *bad, P(fake), ws_n, None) == moe.MOE_ERR_INVALID_ARG


def test_fp8_payload_validates_before_cuda(moe):
    tiny = synth.config("tiny")
    assert moe.moe_check_config(moe.MoeConfig.of(tiny, payload=1)) == moe.MOE_OK
    assert moe.moe_check_config(moe.MoeConfig.of(tiny, payload=2)) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert moe.moe_check_config(moe.MoeConfig.of(tiny.replace(d=192), payload=1)) == \
        moe.MOE_ERR_UNSUPPORTED_SHAPE
    lib, fake, P = moe._lib, 1 << 20, C.c_void_p
    odd = moe.MoeConfig.of(tiny.replace(d=192))          # bf16 payload: fine, but no FP8 entry
    ws_n = moe.moe_workspace_size(odd)
    args = [P(fake)] * 10
    assert lib.moe_dispatch_fp8(C.byref(odd), *args, P(fake), ws_n, None) == \
        moe.MOE_ERR_UNSUPPORTED_SHAPE
    cfg = moe.MoeConfig.of(tiny)
    ws_n = moe.moe_workspace_size(cfg)
    bad = list(args)
    bad[9] = None                                         # x_scale
    assert lib.moe_dispatch_fp8(C.byref(cfg), *bad, P(fake), ws_n, None) == moe.MOE_ERR_INVALID_ARG
    fargs = [P(fake)] * 12
    fargs[1] = P(fake + 4)                                # misaligned scales
    assert lib.moe_expert_ffn_fp8(C.byref(cfg), *fargs, P(fake), ws_n, None) == \
        moe.MOE_ERR_INVALID_ARG


def test_router_variants_validate_before_cuda(moe):
    sh = synth.config("tiny")
    assert moe.moe_check_config(moe.MoeConfig.of(sh, router=3)) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert moe.moe_check_config(moe.MoeConfig.of(sh, router=-1)) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    for r in (moe.MOE_ROUTER_SIGMOID, moe.MOE_ROUTER_SQRT_SOFTPLUS, moe.MOE_ROUTER_HASH):
        assert moe.moe_check_config(moe.MoeConfig.of(sh, router=r)) == moe.MOE_OK
    assert moe.MoeConfig.of(sh).router == moe.MOE_ROUTER_SIGMOID
    lib, fake, P = moe._lib, 1 << 20, C.c_void_p
    hcfg = moe.MoeConfig.of(sh, router=moe.MOE_ROUTER_HASH)
    ws_n = moe.moe_workspace_size(hcfg)
    # the learned router refuses a hash configuration
    assert lib.moe_route(C.byref(hcfg), P(fake), P(fake), None, None, P(fake), P(fake), None,
                         P(fake), ws_n, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_route_hash(C.byref(hcfg), None, None, P(fake), None) == moe.MOE_ERR_INVALID_ARG
    cfg = moe.MoeConfig.of(sh)
    for g in (float("nan"), float("inf"), float("-inf")):
        assert lib.moe_bias_update(C.byref(cfg), P(fake), g, P(fake), None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_bias_update(C.byref(cfg), None, 1e-3, P(fake), None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_bias_update(C.byref(cfg), P(fake), 1e-3, None, None) == moe.MOE_ERR_INVALID_ARG
    # moe_forward: the learned routers need router_w, the hash router does not
    args = [P(fake)] * 18
    args[1] = None  # router_w
    assert lib.moe_forward(C.byref(cfg), *args, P(fake), ws_n, None) == moe.MOE_ERR_INVALID_ARG


def lib_ep_plan_status(moe, cfg, world):
    P = C.c_void_p
    return moe._lib.moe_ep_plan(C.byref(cfg), world, 0, P(1 << 20), P(1 << 20), P(1 << 20), None)


def test_expert_parallel_validates_before_cuda(moe):
    tiny = synth.config("tiny")                        # E = 16, d = 128
    cfg = moe.MoeConfig.of(tiny)
    lib, fake, P = moe._lib, 1 << 20, C.c_void_p
    # world must divide E, 1 <= world <= 64; the workspace is the global batch's
    assert moe.moe_ep_workspace_size(cfg, 3) == 0
    assert moe.moe_ep_workspace_size(cfg, 0) == 0
    assert moe.moe_ep_workspace_size(cfg, 32) == 0
    # world * T * K copies must stay below 2^31 rows at one owner
    big = moe.MoeConfig.of(tiny.replace(T=(1 << 28) - 4))   # T * K just below 2^30
    assert moe.moe_check_config(big) == moe.MOE_OK
    assert lib_ep_plan_status(moe, big, 4) == moe.MOE_ERR_UNSUPPORTED_SHAPE  # 4 T K >= 2^31
    assert moe.moe_ep_workspace_size(big, 4) == 0
    assert moe.moe_ep_workspace_size(cfg, 2) == \
        moe.moe_workspace_size(moe.MoeConfig.of(tiny.replace(T=2 * tiny.T)))
    ws_n = moe.moe_ep_workspace_size(cfg, 2)
    UNS, INV = moe.MOE_ERR_UNSUPPORTED_SHAPE, moe.MOE_ERR_INVALID_ARG
    c = C.byref(cfg)
    assert lib.moe_ep_plan(c, 3, 0, P(fake), P(fake), P(fake), None) == UNS
    assert lib.moe_ep_plan(c, 2, 2, P(fake), P(fake), P(fake), None) == UNS      # rank
    assert lib.moe_ep_plan(c, 2, 0, None, P(fake), P(fake), None) == INV
    d_args = [P(fake)] * 6                     # x, topk_idx, offsets, inv_perm, base, recv_x
    bad = list(d_args)
    bad[5] = None
    assert lib.moe_ep_dispatch(c, 2, *bad, None, None) == INV
    bad = list(d_args)
    bad[0] = P(fake + 8)                       # misaligned x
    assert lib.moe_ep_dispatch(c, 2, *bad, None, None) == INV
    assert lib.moe_ep_dispatch(c, 5, *d_args, None, None) == UNS
    odd = moe.MoeConfig.of(tiny.replace(d=192))
    q_args = [P(fake)] * 7                     # ..., recv_q, recv_scale
    assert lib.moe_ep_dispatch_fp8(C.byref(odd), 2, *q_args, None, None) == UNS
    bad = list(q_args)
    bad[6] = None
    assert lib.moe_ep_dispatch_fp8(c, 2, *bad, None, None) == INV
    f_args = [P(fake)] * 11                    # recv_x .. y_shared
    assert lib.moe_ep_expert_ffn(c, 2, 0, *f_args, P(fake), ws_n - 1, None) == \
        moe.MOE_ERR_WORKSPACE_TOO_SMALL
    assert lib.moe_ep_expert_ffn(c, 2, -1, *f_args, P(fake), ws_n, None) == UNS
    bad = list(f_args)
    bad[0] = None                              # recv_x
    assert lib.moe_ep_expert_ffn(c, 2, 0, *bad, P(fake), ws_n, None) == INV
    assert lib.moe_ep_expert_ffn(c, 2, 0, *f_args, P(fake + 16), ws_n, None) == INV  # ws align
    g_args = [P(fake)] * 12                    # recv_q, recv_scale, ... y_shared
    bad = list(g_args)
    bad[1] = None                              # recv_scale
    assert lib.moe_ep_expert_ffn_fp8(c, 2, 0, *bad, P(fake), ws_n, None) == INV
    bad = list(g_args)
    bad[1] = P(fake + 4)                       # misaligned scales
    assert lib.moe_ep_expert_ffn_fp8(c, 2, 0, *bad, P(fake), ws_n, None) == INV
    assert lib.moe_ep_expert_ffn_fp8(C.byref(odd), 2, 0, *g_args, P(fake), ws_n, None) == UNS
    c_args = [P(fake)] * 7                     # topk_idx .. y_shared, then out
    assert lib.moe_ep_combine(c, 2, *c_args, None, None, None) == INV         # out
    bad = list(c_args)
    bad[6] = P(fake + 2)                       # misaligned y_shared
    assert lib.moe_ep_combine(c, 2, *bad, P(fake), None, None) == INV
    assert lib.moe_ep_token_plan(c, 3, P(fake), P(fake), P(fake), None) == UNS
    assert lib.moe_ep_token_plan(c, 2, None, P(fake), P(fake), None) == INV
    assert lib.moe_ep_token_base(c, 2, 2, P(fake), P(fake), None) == UNS
    assert lib.moe_ep_token_base(c, 2, 0, P(fake), None, None) == INV
    dd_args = [P(fake)] * 9                    # x .. tok_base, recv_tok, recv_idx
    bad = list(dd_args)
    bad[8] = None                              # recv_idx
    assert lib.moe_ep_dispatch_dedup(c, 2, *bad, None, None) == INV
    bad = list(dd_args)
    bad[0] = P(fake + 8)                       # misaligned x
    assert lib.moe_ep_dispatch_dedup(c, 2, *bad, None, None) == INV
    assert lib.moe_ep_fanout(c, 2, P(fake), P(fake), None, P(fake), None, None) == INV
    assert lib.moe_ep_fanout(c, 2, P(fake + 4), P(fake), P(fake), P(fake), None, None) == INV
    assert lib.moe_ep_fanout(c, 3, P(fake), P(fake), P(fake), P(fake), None, None) == UNS
    dq_args = [P(fake)] * 10                   # x .. tok_base, recv_tq, recv_ts, recv_idx
    assert lib.moe_ep_dispatch_dedup_fp8(C.byref(odd), 2, *dq_args, None, None) == UNS
    bad = list(dq_args)
    bad[8] = None                              # recv_ts
    assert lib.moe_ep_dispatch_dedup_fp8(c, 2, *bad, None, None) == INV
    fq_args = [P(fake)] * 6                    # recv_tq, recv_ts, recv_idx, loff, recv_q, scale
    assert lib.moe_ep_fanout_fp8(C.byref(odd), 2, *fq_args, None, None) == UNS
    bad = list(fq_args)
    bad[4] = P(fake + 8)                       # misaligned recv_q
    assert lib.moe_ep_fanout_fp8(c, 2, *bad, None, None) == INV
    cp_args = [P(fake)] * 10                   # topk_idx .. lcnt
    bad = list(cp_args)
    bad[9] = None                              # lcnt
    assert lib.moe_ep_combine_plan(c, 2, *bad, None, None) == INV
    assert lib.moe_ep_combine_plan(c, 3, *cp_args, None, None) == UNS
    # dispatch + combine lists in one launch: x, topk_idx, topk_w, offsets, inv_perm, base,
    # tok_slot, tok_base, recv_tok, recv_idx, list, lw, lcnt
    dp_args = [P(fake)] * 13
    for i in (2, 10, 12):                      # topk_w, list, lcnt
        bad = list(dp_args)
        bad[i] = None
        assert lib.moe_ep_dispatch_dedup_plan(c, 2, *bad, None, None) == INV
    bad = list(dp_args)
    bad[0] = P(fake + 8)                       # misaligned x
    assert lib.moe_ep_dispatch_dedup_plan(c, 2, *bad, None, None) == INV
    assert lib.moe_ep_dispatch_dedup_plan(c, 3, *dp_args, None, None) == UNS
    pc_args = [P(fake)] * 6                    # recv_y, list, lw, lcnt, tok_base, partial
    bad = list(pc_args)
    bad[5] = P(fake + 8)                       # misaligned partial
    assert lib.moe_ep_precombine(c, 2, *bad, None, None) == INV
    bad = list(pc_args)
    bad[1] = None                              # list
    assert lib.moe_ep_precombine(c, 2, *bad, None, None) == INV
    cd_args = [P(fake)] * 6                    # topk_idx, tok_slot, tok_base, partial, y_sh, out
    bad = list(cd_args)
    bad[5] = None                              # out
    assert lib.moe_ep_combine_dedup(c, 2, *bad, None, None) == INV
    bad = list(cd_args)
    bad[4] = P(fake + 2)                       # misaligned y_shared
    assert lib.moe_ep_combine_dedup(c, 2, *bad, None, None) == INV
    assert lib.moe_ipc_get_handle(None, P(fake)) == INV
    assert lib.moe_ipc_open_handle(None, P(fake)) == INV
    assert lib.moe_ipc_close_handle(None) == INV


@pytest.mark.skipif(torch.cuda.is_available(), reason="needs a machine without a GPU")
def test_no_device_is_reported(moe):
    assert moe._lib.moe_clear_device_status(C.c_void_p(1 << 20), None) == moe.MOE_ERR_NO_DEVICE
    assert moe._lib.moe_last_device_status(C.c_void_p(1 << 20), None) == moe.MOE_ERR_NO_DEVICE
    assert moe._lib.moe_last_device_status(None, None) == moe.MOE_ERR_INVALID_ARG
