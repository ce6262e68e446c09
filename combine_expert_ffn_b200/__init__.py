"""Python binding of libmoe, the B200 (sm_100a) MoE-layer forward library.

Argument marshalling only: every function below forwards torch tensors'
device pointers and the current CUDA stream to the C entry point of the same
name in ``include/moe.h`` and raises :class:`MoeError` on a nonzero status.
All arithmetic happens in the library's CUDA kernels; there is no CPU or
PyTorch fallback.  If ``libmoe.so`` is missing the import fails -- build it
with ``python combine_expert_ffn_b200/build.py``.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: run `python combine_expert_ffn_b200/build.py`")

_lib = C.CDLL(LIB_PATH)

STATUS = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE",
    3: "MOE_ERR_WORKSPACE_TOO_SMALL", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_TIMEOUT",
    6: "MOE_ERR_DEVICE_FAULT", 7: "MOE_ERR_NO_DEVICE",
}
MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED_SHAPE, MOE_ERR_WORKSPACE_TOO_SMALL, \
    MOE_ERR_CUDA, MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_DEVICE_FAULT, MOE_ERR_NO_DEVICE = range(8)

EXPORTS = ("moe_check_config", "moe_workspace_size", "moe_status_string", "moe_launch_count",
           "moe_read_device_status", "moe_last_device_status", "moe_clear_device_status",
           "moe_route", "moe_route_select",
           "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_forward",
           "moe_selftest_bounded_wait", "moe_dispatch_noalloc", "moe_route_hash",
           "moe_bias_update", "moe_expert_ffn_gather", "moe_dispatch_fp8",
           "moe_expert_ffn_fp8", "moe_permute", "moe_ep_workspace_size", "moe_ep_plan",
           "moe_ep_dispatch", "moe_ep_expert_ffn", "moe_ep_combine", "moe_ep_dispatch_fp8",
           "moe_ep_expert_ffn_fp8", "moe_ep_token_plan", "moe_ep_token_base",
           "moe_ep_dispatch_dedup", "moe_ep_fanout", "moe_ep_dispatch_dedup_fp8",
           "moe_ep_fanout_fp8", "moe_ep_combine_plan", "moe_ep_dispatch_dedup_plan",
           "moe_ep_precombine", "moe_ep_combine_dedup", "moe_ipc_get_handle",
           "moe_ipc_open_handle", "moe_ipc_close_handle", "moe_packed_weights_size",
           "moe_pack_weights", "moe_expert_ffn_packed", "moe_forward_packed")

MOE_ROUTER_SIGMOID, MOE_ROUTER_SQRT_SOFTPLUS, MOE_ROUTER_HASH = 0, 1, 2
MOE_PAYLOAD_BF16, MOE_PAYLOAD_FP8 = 0, 1


class MoeConfig(C.Structure):
    """Mirror of ``moe_config``."""
    _fields_ = [(n, C.c_int32) for n in
                ("T", "d", "E", "G", "K", "M", "d_ff", "n_shared", "d_ff_shared", "router",
                 "payload")]

    @classmethod
    def of(cls, shape, router=None, payload=None) -> "MoeConfig":
        """From any object with the nine size attributes (e.g. ``synth.MoeShape``);
        router and payload from the arguments, else the object's, else the defaults
        (sigmoid router, bf16 payload)."""
        if router is None:
            router = getattr(shape, "router", MOE_ROUTER_SIGMOID)
        if payload is None:
            payload = getattr(shape, "payload", MOE_PAYLOAD_BF16)
        return cls(*(int(getattr(shape, n)) for n, _ in cls._fields_[:-2]), int(router),
                   int(payload))

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


class MoeError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn}: {STATUS.get(status, status)} ({moe_status_string(status)})")


_P, _S, _I64 = C.c_void_p, C.c_size_t, C.c_int64
_CP = C.POINTER(MoeConfig)
_sig = {
    "moe_check_config": (C.c_int, [_CP]),
    "moe_workspace_size": (_S, [_CP]),
    "moe_status_string": (C.c_char_p, [C.c_int]),
    "moe_launch_count": (C.c_uint64, []),
    "moe_read_device_status": (C.c_int, [_P, _P, _P]),
    "moe_last_device_status": (C.c_int, [_P, _P]),
    "moe_clear_device_status": (C.c_int, [_P, _P]),
    "moe_route": (C.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]),
    "moe_route_select": (C.c_int, [_CP, _P, _P, _P, _P, _P]),
    "moe_dispatch": (C.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]),
    "moe_expert_ffn": (C.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]),
    "moe_combine": (C.c_int, [_CP, _P, _P, _P, _P, _P, _P]),
    "moe_forward": (C.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                              _P, _P, _P, _P, _P, _S, _P]),
    "moe_route_hash": (C.c_int, [_CP, _P, _P, _P, _P]),
    "moe_permute": (C.c_int, [_CP, _P, _P, _P, _P]),
    "moe_ep_workspace_size": (_S, [_CP, C.c_int32]),
    "moe_ep_plan": (C.c_int, [_CP, C.c_int32, C.c_int32, _P, _P, _P, _P]),
    "moe_ep_dispatch": (C.c_int, [_CP, C.c_int32, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_ep_expert_ffn": (C.c_int, [_CP, C.c_int32, C.c_int32, _P, _P, _P, _P, _P, _P, _P, _P,
                                    _P, _P, _P, _P, _S, _P]),
    "moe_ep_combine": (C.c_int, [_CP, C.c_int32, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_ep_token_plan": (C.c_int, [_CP, C.c_int32, _P, _P, _P, _P]),
    "moe_ep_token_base": (C.c_int, [_CP, C.c_int32, C.c_int32, _P, _P, _P]),
    "moe_ep_dispatch_dedup": (C.c_int, [_CP, C.c_int32] + [_P] * 11),
    "moe_ep_fanout": (C.c_int, [_CP, C.c_int32] + [_P] * 6),
    "moe_ep_dispatch_dedup_fp8": (C.c_int, [_CP, C.c_int32] + [_P] * 12),
    "moe_ep_fanout_fp8": (C.c_int, [_CP, C.c_int32] + [_P] * 8),
    "moe_ep_combine_plan": (C.c_int, [_CP, C.c_int32] + [_P] * 12),
    "moe_ep_dispatch_dedup_plan": (C.c_int, [_CP, C.c_int32] + [_P] * 15),
    "moe_ep_precombine": (C.c_int, [_CP, C.c_int32] + [_P] * 8),
    "moe_ep_combine_dedup": (C.c_int, [_CP, C.c_int32] + [_P] * 8),
    "moe_ep_dispatch_fp8": (C.c_int, [_CP, C.c_int32, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_ep_expert_ffn_fp8": (C.c_int, [_CP, C.c_int32, C.c_int32, _P, _P, _P, _P, _P, _P, _P,
                                        _P, _P, _P, _P, _P, _P, _S, _P]),
    "moe_ipc_get_handle": (C.c_int, [_P, _P]),
    "moe_ipc_open_handle": (C.c_int, [_P, _P]),
    "moe_ipc_close_handle": (C.c_int, [_P]),
    "moe_dispatch_fp8": (C.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]),
    "moe_expert_ffn_fp8": (C.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S,
                                     _P]),
    "moe_expert_ffn_gather": (C.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S,
                                        _P]),
    "moe_bias_update": (C.c_int, [_CP, _P, C.c_float, _P, _P]),
    "moe_selftest_bounded_wait": (C.c_int, [_I64, _P, _P]),
    "moe_dispatch_noalloc": (C.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_packed_weights_size": (_S, [_CP]),
    "moe_pack_weights": (C.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_expert_ffn_packed": (C.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _S, _P]),
    "moe_forward_packed": (C.c_int, [_CP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                     _P, _S, _P]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _cfg(cfg):
    return C.byref(cfg if isinstance(cfg, MoeConfig) else MoeConfig.of(cfg))


def _ok(fn, st):
    if st != MOE_OK:
        raise MoeError(fn, st)


def _ws(ws):
    return (None, 0) if ws is None else (ws.data_ptr(), ws.numel() * ws.element_size())


# ----------------------------------------------------------------- queries
def moe_check_config(cfg) -> int:
    return _lib.moe_check_config(_cfg(cfg))


def moe_workspace_size(cfg) -> int:
    return _lib.moe_workspace_size(_cfg(cfg))


def moe_status_string(status: int) -> str:
    return _lib.moe_status_string(int(status)).decode()


def moe_launch_count() -> int:
    return _lib.moe_launch_count()


def alloc_workspace(cfg, device="cuda") -> torch.Tensor:
    """Device workspace of moe_workspace_size(cfg) bytes (torch blocks are 512-byte aligned)."""
    n = moe_workspace_size(cfg)
    if n == 0:
        raise MoeError("moe_workspace_size", moe_check_config(cfg) or MOE_ERR_UNSUPPORTED_SHAPE)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def moe_read_device_status(ws, stream=None) -> int:
    out = C.c_int32(-1)
    _ok("moe_read_device_status", _lib.moe_read_device_status(_ptr(ws), C.byref(out), _stream(stream)))
    return out.value


def moe_last_device_status(ws, stream=None) -> int:
    """The device status word (synchronises the stream); host-side read errors as codes."""
    return int(_lib.moe_last_device_status(_ptr(ws), _stream(stream)))


def moe_clear_device_status(ws, stream=None) -> None:
    _ok("moe_clear_device_status", _lib.moe_clear_device_status(_ptr(ws), _stream(stream)))


# ----------------------------------------------------------------- stages
def moe_route(cfg, x, router_w, logit_offset, bias, topk_idx, topk_w, scores=None, ws=None,
              stream=None) -> None:
    wp, wn = _ws(ws)
    _ok("moe_route", _lib.moe_route(_cfg(cfg), _ptr(x), _ptr(router_w), _ptr(logit_offset),
                                    _ptr(bias), _ptr(topk_idx), _ptr(topk_w), _ptr(scores), wp, wn,
                                    _stream(stream)))


def moe_route_hash(cfg, token_ids, topk_idx, topk_w, stream=None) -> None:
    _ok("moe_route_hash", _lib.moe_route_hash(_cfg(cfg), _ptr(token_ids), _ptr(topk_idx),
                                              _ptr(topk_w), _stream(stream)))


def moe_bias_update(cfg, counts, gamma, bias, stream=None) -> None:
    _ok("moe_bias_update", _lib.moe_bias_update(_cfg(cfg), _ptr(counts), C.c_float(gamma),
                                                _ptr(bias), _stream(stream)))


def moe_route_select(cfg, scores, bias, topk_idx, topk_w, stream=None) -> None:
    _ok("moe_route_select", _lib.moe_route_select(_cfg(cfg), _ptr(scores), _ptr(bias),
                                                  _ptr(topk_idx), _ptr(topk_w), _stream(stream)))


def moe_dispatch(cfg, x, topk_idx, counts, offsets, send, send_tok, perm_token, inv_perm, x_perm,
                 ws, stream=None) -> None:
    wp, wn = _ws(ws)
    _ok("moe_dispatch", _lib.moe_dispatch(_cfg(cfg), _ptr(x), _ptr(topk_idx), _ptr(counts),
                                          _ptr(offsets), _ptr(send), _ptr(send_tok),
                                          _ptr(perm_token), _ptr(inv_perm), _ptr(x_perm), wp, wn,
                                          _stream(stream)))


def moe_expert_ffn(cfg, x_perm, offsets, w_gate, w_up, w_down, y_perm, x, ws_gate, ws_up, ws_down,
                   y_shared, ws, stream=None) -> None:
    wp, wn = _ws(ws)
    _ok("moe_expert_ffn", _lib.moe_expert_ffn(_cfg(cfg), _ptr(x_perm), _ptr(offsets), _ptr(w_gate),
                                              _ptr(w_up), _ptr(w_down), _ptr(y_perm), _ptr(x),
                                              _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down),
                                              _ptr(y_shared), wp, wn, _stream(stream)))


def moe_expert_ffn_gather(cfg, x, perm_token, offsets, w_gate, w_up, w_down, y_perm, ws_gate,
                          ws_up, ws_down, y_shared, ws, stream=None) -> None:
    wp, wn = _ws(ws)
    _ok("moe_expert_ffn_gather",
        _lib.moe_expert_ffn_gather(_cfg(cfg), _ptr(x), _ptr(perm_token), _ptr(offsets),
                                   _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(y_perm),
                                   _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(y_shared), wp,
                                   wn, _stream(stream)))


def moe_permute(cfg, x, inv_perm, x_perm, stream=None) -> None:
    _ok("moe_permute", _lib.moe_permute(_cfg(cfg), _ptr(x), _ptr(inv_perm), _ptr(x_perm),
                                        _stream(stream)))


# ----------------------------------------------------------------- expert parallelism
def moe_ep_workspace_size(cfg, world) -> int:
    return _lib.moe_ep_workspace_size(_cfg(cfg), int(world))


def moe_ep_plan(cfg, world, rank, counts_all, base, local_offsets, stream=None) -> None:
    _ok("moe_ep_plan", _lib.moe_ep_plan(_cfg(cfg), int(world), int(rank), _ptr(counts_all),
                                        _ptr(base), _ptr(local_offsets), _stream(stream)))


def moe_ep_dispatch(cfg, world, x, topk_idx, offsets, inv_perm, base, recv_x_ptrs,
                    device_status=None, stream=None) -> None:
    """recv_x_ptrs: device int64 tensor of `world` device pointers."""
    _ok("moe_ep_dispatch",
        _lib.moe_ep_dispatch(_cfg(cfg), int(world), _ptr(x), _ptr(topk_idx), _ptr(offsets),
                             _ptr(inv_perm), _ptr(base), _ptr(recv_x_ptrs), _ptr(device_status),
                             _stream(stream)))


def moe_ep_expert_ffn(cfg, world, rank, recv_x, local_offsets, w_gate, w_up, w_down, recv_y, x,
                      ws_gate, ws_up, ws_down, y_shared, ws, stream=None) -> None:
    wp, wn = _ws(ws)
    _ok("moe_ep_expert_ffn",
        _lib.moe_ep_expert_ffn(_cfg(cfg), int(world), int(rank), _ptr(recv_x),
                               _ptr(local_offsets), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                               _ptr(recv_y), _ptr(x), _ptr(ws_gate), _ptr(ws_up),
                               _ptr(ws_down), _ptr(y_shared), wp, wn, _stream(stream)))


def moe_ep_token_plan(cfg, world, topk_idx, tok_slot, tok_counts, stream=None) -> None:
    _ok("moe_ep_token_plan",
        _lib.moe_ep_token_plan(_cfg(cfg), int(world), _ptr(topk_idx), _ptr(tok_slot),
                               _ptr(tok_counts), _stream(stream)))


def moe_ep_token_base(cfg, world, rank, tok_counts_all, tok_base, stream=None) -> None:
    _ok("moe_ep_token_base",
        _lib.moe_ep_token_base(_cfg(cfg), int(world), int(rank), _ptr(tok_counts_all),
                               _ptr(tok_base), _stream(stream)))


def moe_ep_dispatch_dedup(cfg, world, x, topk_idx, offsets, inv_perm, base, tok_slot, tok_base,
                          recv_tok_ptrs, recv_idx_ptrs, device_status=None, stream=None) -> None:
    """recv_tok_ptrs / recv_idx_ptrs: device int64 tensors of `world` device pointers."""
    _ok("moe_ep_dispatch_dedup",
        _lib.moe_ep_dispatch_dedup(_cfg(cfg), int(world), _ptr(x), _ptr(topk_idx), _ptr(offsets),
                                   _ptr(inv_perm), _ptr(base), _ptr(tok_slot), _ptr(tok_base),
                                   _ptr(recv_tok_ptrs), _ptr(recv_idx_ptrs), _ptr(device_status),
                                   _stream(stream)))


def moe_ep_fanout(cfg, world, recv_tok, recv_idx, local_offsets, recv_x, device_status=None,
                  stream=None) -> None:
    _ok("moe_ep_fanout",
        _lib.moe_ep_fanout(_cfg(cfg), int(world), _ptr(recv_tok), _ptr(recv_idx),
                           _ptr(local_offsets), _ptr(recv_x), _ptr(device_status),
                           _stream(stream)))


def moe_ep_dispatch_dedup_fp8(cfg, world, x, topk_idx, offsets, inv_perm, base, tok_slot,
                              tok_base, recv_tq_ptrs, recv_ts_ptrs, recv_idx_ptrs,
                              device_status=None, stream=None) -> None:
    _ok("moe_ep_dispatch_dedup_fp8",
        _lib.moe_ep_dispatch_dedup_fp8(_cfg(cfg), int(world), _ptr(x), _ptr(topk_idx),
                                       _ptr(offsets), _ptr(inv_perm), _ptr(base), _ptr(tok_slot),
                                       _ptr(tok_base), _ptr(recv_tq_ptrs), _ptr(recv_ts_ptrs),
                                       _ptr(recv_idx_ptrs), _ptr(device_status), _stream(stream)))


def moe_ep_fanout_fp8(cfg, world, recv_tq, recv_ts, recv_idx, local_offsets, recv_q, recv_scale,
                      device_status=None, stream=None) -> None:
    _ok("moe_ep_fanout_fp8",
        _lib.moe_ep_fanout_fp8(_cfg(cfg), int(world), _ptr(recv_tq), _ptr(recv_ts),
                               _ptr(recv_idx), _ptr(local_offsets), _ptr(recv_q),
                               _ptr(recv_scale), _ptr(device_status), _stream(stream)))


def moe_ep_combine_plan(cfg, world, topk_idx, topk_w, offsets, inv_perm, base, tok_slot, tok_base,
                        list_ptrs, lw_ptrs, lcnt_ptrs, device_status=None, stream=None) -> None:
    _ok("moe_ep_combine_plan",
        _lib.moe_ep_combine_plan(_cfg(cfg), int(world), _ptr(topk_idx), _ptr(topk_w),
                                 _ptr(offsets), _ptr(inv_perm), _ptr(base), _ptr(tok_slot),
                                 _ptr(tok_base), _ptr(list_ptrs), _ptr(lw_ptrs), _ptr(lcnt_ptrs),
                                 _ptr(device_status), _stream(stream)))


def moe_ep_dispatch_dedup_plan(cfg, world, x, topk_idx, topk_w, offsets, inv_perm, base,
                               tok_slot, tok_base, recv_tok_ptrs, recv_idx_ptrs, list_ptrs,
                               lw_ptrs, lcnt_ptrs, device_status=None, stream=None) -> None:
    """moe_ep_dispatch_dedup + moe_ep_combine_plan in one launch (same outputs)."""
    _ok("moe_ep_dispatch_dedup_plan",
        _lib.moe_ep_dispatch_dedup_plan(_cfg(cfg), int(world), _ptr(x), _ptr(topk_idx),
                                        _ptr(topk_w), _ptr(offsets), _ptr(inv_perm), _ptr(base),
                                        _ptr(tok_slot), _ptr(tok_base), _ptr(recv_tok_ptrs),
                                        _ptr(recv_idx_ptrs), _ptr(list_ptrs), _ptr(lw_ptrs),
                                        _ptr(lcnt_ptrs), _ptr(device_status), _stream(stream)))


def moe_ep_precombine(cfg, world, recv_y, lst, lw, lcnt, tok_base, partial, device_status=None,
                      stream=None) -> None:
    _ok("moe_ep_precombine",
        _lib.moe_ep_precombine(_cfg(cfg), int(world), _ptr(recv_y), _ptr(lst), _ptr(lw),
                               _ptr(lcnt), _ptr(tok_base), _ptr(partial), _ptr(device_status),
                               _stream(stream)))


def moe_ep_combine_dedup(cfg, world, topk_idx, tok_slot, tok_base, partial_ptrs, y_shared, out,
                         device_status=None, stream=None) -> None:
    _ok("moe_ep_combine_dedup",
        _lib.moe_ep_combine_dedup(_cfg(cfg), int(world), _ptr(topk_idx), _ptr(tok_slot),
                                  _ptr(tok_base), _ptr(partial_ptrs), _ptr(y_shared), _ptr(out),
                                  _ptr(device_status), _stream(stream)))


def moe_ep_dispatch_fp8(cfg, world, x, topk_idx, offsets, inv_perm, base, recv_q_ptrs,
                        recv_scale_ptrs, device_status=None, stream=None) -> None:
    """recv_q_ptrs / recv_scale_ptrs: device int64 tensors of `world` device pointers."""
    _ok("moe_ep_dispatch_fp8",
        _lib.moe_ep_dispatch_fp8(_cfg(cfg), int(world), _ptr(x), _ptr(topk_idx), _ptr(offsets),
                                 _ptr(inv_perm), _ptr(base), _ptr(recv_q_ptrs),
                                 _ptr(recv_scale_ptrs), _ptr(device_status), _stream(stream)))


def moe_ep_expert_ffn_fp8(cfg, world, rank, recv_q, recv_scale, local_offsets, w_gate, w_up,
                          w_down, recv_y, x, ws_gate, ws_up, ws_down, y_shared, ws,
                          stream=None) -> None:
    wp, wn = _ws(ws)
    _ok("moe_ep_expert_ffn_fp8",
        _lib.moe_ep_expert_ffn_fp8(_cfg(cfg), int(world), int(rank), _ptr(recv_q),
                                   _ptr(recv_scale), _ptr(local_offsets), _ptr(w_gate),
                                   _ptr(w_up), _ptr(w_down), _ptr(recv_y), _ptr(x),
                                   _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(y_shared), wp,
                                   wn, _stream(stream)))


def moe_ep_combine(cfg, world, topk_idx, topk_w, offsets, inv_perm, base, recv_y_ptrs, y_shared,
                   out, device_status=None, stream=None) -> None:
    _ok("moe_ep_combine",
        _lib.moe_ep_combine(_cfg(cfg), int(world), _ptr(topk_idx), _ptr(topk_w), _ptr(offsets),
                            _ptr(inv_perm), _ptr(base), _ptr(recv_y_ptrs), _ptr(y_shared),
                            _ptr(out), _ptr(device_status), _stream(stream)))


MOE_IPC_HANDLE_BYTES = 72


def moe_ipc_get_handle(t) -> bytes:
    h = (C.c_char * MOE_IPC_HANDLE_BYTES)()
    _ok("moe_ipc_get_handle", _lib.moe_ipc_get_handle(_ptr(t), C.cast(h, C.c_void_p)))
    return bytes(h)


def moe_ipc_open_handle(handle: bytes) -> int:
    buf = (C.c_char * MOE_IPC_HANDLE_BYTES).from_buffer_copy(handle)
    p = C.c_void_p()
    _ok("moe_ipc_open_handle", _lib.moe_ipc_open_handle(C.cast(buf, C.c_void_p), C.byref(p)))
    return p.value


def moe_ipc_close_handle(ptr: int) -> None:
    _ok("moe_ipc_close_handle", _lib.moe_ipc_close_handle(C.c_void_p(ptr)))


def moe_dispatch_fp8(cfg, x, topk_idx, counts, offsets, send, send_tok, perm_token, inv_perm,
                     x_perm_q, x_scale, ws, stream=None) -> None:
    wp, wn = _ws(ws)
    _ok("moe_dispatch_fp8",
        _lib.moe_dispatch_fp8(_cfg(cfg), _ptr(x), _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                              _ptr(send), _ptr(send_tok), _ptr(perm_token), _ptr(inv_perm),
                              _ptr(x_perm_q), _ptr(x_scale), wp, wn, _stream(stream)))


def moe_expert_ffn_fp8(cfg, x_perm_q, x_scale, offsets, w_gate, w_up, w_down, y_perm, x, ws_gate,
                       ws_up, ws_down, y_shared, ws, stream=None) -> None:
    wp, wn = _ws(ws)
    _ok("moe_expert_ffn_fp8",
        _lib.moe_expert_ffn_fp8(_cfg(cfg), _ptr(x_perm_q), _ptr(x_scale), _ptr(offsets),
                                _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(y_perm), _ptr(x),
                                _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(y_shared), wp, wn,
                                _stream(stream)))


def moe_combine(cfg, y_perm, inv_perm, topk_w, y_shared, out, stream=None) -> None:
    _ok("moe_combine", _lib.moe_combine(_cfg(cfg), _ptr(y_perm), _ptr(inv_perm), _ptr(topk_w),
                                        _ptr(y_shared), _ptr(out), _stream(stream)))


def moe_forward(cfg, x, router_w, logit_offset, bias, w_gate, w_up, w_down, ws_gate, ws_up,
                ws_down, out, topk_idx=None, topk_w=None, counts=None, offsets=None, send=None,
                send_tok=None, ws=None, stream=None, token_ids=None) -> None:
    wp, wn = _ws(ws)
    _ok("moe_forward", _lib.moe_forward(_cfg(cfg), _ptr(x), _ptr(router_w), _ptr(logit_offset),
                                        _ptr(bias), _ptr(token_ids), _ptr(w_gate), _ptr(w_up),
                                        _ptr(w_down),
                                        _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(out),
                                        _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(offsets),
                                        _ptr(send), _ptr(send_tok), wp, wn, _stream(stream)))


def moe_packed_weights_size(cfg) -> int:
    return int(_lib.moe_packed_weights_size(_cfg(cfg)))


def moe_pack_weights(cfg, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, packed,
                     stream=None) -> None:
    _ok("moe_pack_weights", _lib.moe_pack_weights(_cfg(cfg), _ptr(w_gate), _ptr(w_up),
                                                  _ptr(w_down), _ptr(ws_gate), _ptr(ws_up),
                                                  _ptr(ws_down), _ptr(packed), _stream(stream)))


def pack_weights(cfg, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, device="cuda",
                 stream=None):
    """Allocates the packed-weight buffer (uint8) and fills it with moe_pack_weights."""
    n = moe_packed_weights_size(cfg)
    if n == 0:
        raise MoeError("moe_packed_weights_size", MOE_ERR_UNSUPPORTED_SHAPE)
    packed = torch.empty(n, dtype=torch.uint8, device=device)
    moe_pack_weights(cfg, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, packed, stream)
    return packed


def moe_expert_ffn_packed(cfg, x_perm, offsets, packed, y_perm, x, y_shared, ws,
                          stream=None) -> None:
    wp, wn = _ws(ws)
    _ok("moe_expert_ffn_packed",
        _lib.moe_expert_ffn_packed(_cfg(cfg), _ptr(x_perm), _ptr(offsets), _ptr(packed),
                                   _ptr(y_perm), _ptr(x), _ptr(y_shared), wp, wn,
                                   _stream(stream)))


def moe_forward_packed(cfg, x, router_w, logit_offset, bias, packed, out, topk_idx=None,
                       topk_w=None, counts=None, offsets=None, send=None, send_tok=None, ws=None,
                       stream=None, token_ids=None) -> None:
    wp, wn = _ws(ws)
    _ok("moe_forward_packed",
        _lib.moe_forward_packed(_cfg(cfg), _ptr(x), _ptr(router_w), _ptr(logit_offset),
                                _ptr(bias), _ptr(token_ids), _ptr(packed), _ptr(out),
                                _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(offsets),
                                _ptr(send), _ptr(send_tok), wp, wn, _stream(stream)))


def moe_selftest_bounded_wait(timeout_ns, ws, stream=None) -> None:
    _ok("moe_selftest_bounded_wait",
        _lib.moe_selftest_bounded_wait(int(timeout_ns), _ptr(ws), _stream(stream)))


def moe_dispatch_noalloc(cfg, x, topk_idx, counts, offsets, send, send_tok, perm_token, inv_perm,
                         x_perm, device_status=None, stream=None) -> None:
    """moe_dispatch with its scratch in the library's static device array (no workspace)."""
    _ok("moe_dispatch_noalloc",
        _lib.moe_dispatch_noalloc(_cfg(cfg), _ptr(x), _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                                  _ptr(send), _ptr(send_tok), _ptr(perm_token), _ptr(inv_perm),
                                  _ptr(x_perm), _ptr(device_status), _stream(stream)))


# ----------------------------------------------------------------- convenience
def forward_outputs(cfg, device="cuda"):
    """Allocates the outputs of moe_forward (out, topk_idx, topk_w, counts, offsets, send, send_tok)."""
    c = cfg if isinstance(cfg, MoeConfig) else MoeConfig.of(cfg)
    return {
        "out": torch.empty(c.T, c.d, dtype=torch.bfloat16, device=device),
        "topk_idx": torch.empty(c.T, c.K, dtype=torch.int32, device=device),
        "topk_w": torch.empty(c.T, c.K, dtype=torch.float32, device=device),
        "counts": torch.empty(c.E, dtype=torch.int32, device=device),
        "offsets": torch.empty(c.E + 1, dtype=torch.int32, device=device),
        "send": torch.empty(c.G, c.G, dtype=torch.int32, device=device),
        "send_tok": torch.empty(c.G, c.G, dtype=torch.int32, device=device),
    }
