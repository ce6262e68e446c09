"""ctypes binding of the plain C MoE-layer oracle (``moe_oracle.c``).

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  It shares nothing with
the CUDA path; it takes and returns host (CPU) arrays only.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

OK, EBADARG, EINDEX, ENOMEM = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile the oracle with plain IEEE semantics (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
               "-shared", "-Wall", "-Wextra", "-pthread", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        P = C.c_void_p
        i32, i64 = C.c_int, C.c_int64
        _lib.oracle_router_scores.argtypes = [i32, P, i32, i32, P, P, P, P]
        _lib.oracle_select.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P]
        _lib.oracle_dispatch.argtypes = [i32, i32, i32, i32, P, P, P, P, P, P, P]
        _lib.oracle_ffn_row.argtypes = [i32, i32, P, P, P, P, i32, P]
        _lib.oracle_shared_row.argtypes = [i32, i32, i32, P, P, P, P, i32, P]
        _lib.oracle_combine.argtypes = [i32, i32, i32, i64, P, P, P, P, P]
        _lib.oracle_layer_rows.argtypes = [i32, P, i32, i32, i32, i32, i32, i32, i32, i32,
                                           P, P, P, P, P, P, P, P, P, P, i32, P, P, P, P]
        _lib.oracle_router_affinity.argtypes = [i32, P, i32, i32, P, P, P, i32, P]
        _lib.oracle_layer_rows_ex.argtypes = [i32, P, i32, i32, i32, i32, i32, i32, i32, i32,
                                              P, P, P, P, i32, P, i32, P, P, P, P, P, P, i32, P,
                                              P, P, P]
        _lib.oracle_layer_rows_mt.argtypes = [i32] + _lib.oracle_layer_rows_ex.argtypes
        _lib.oracle_e4m3_decode.argtypes = [C.c_uint8]
        _lib.oracle_e4m3_decode.restype = C.c_double
        _lib.oracle_e4m3_encode.argtypes = [C.c_float]
        _lib.oracle_e4m3_encode.restype = C.c_uint8
        _lib.oracle_fp8_quantize_row.argtypes = [i32, P, P, P]
        _lib.oracle_ep_plan.argtypes = [i32, i32, P, P, P]
        _lib.oracle_ep_token_plan.argtypes = [i32, i32, i32, i32, P, P, P]
        _lib.oracle_ep_token_base.argtypes = [i32, P, P]
        _lib.oracle_fp8_dequantize_row.argtypes = [i32, P, P, P]
        _lib.oracle_hash_route.argtypes = [i32, P, i32, i32, i32, i32, P, P]
        _lib.oracle_lowbias32.argtypes = [C.c_uint32]
        _lib.oracle_lowbias32.restype = C.c_uint32
        _lib.oracle_bias_update.argtypes = [i32, i32, i32, P, C.c_float, P]
        for f in ("oracle_router_scores", "oracle_select", "oracle_dispatch",
                  "oracle_ffn_row", "oracle_shared_row", "oracle_combine",
                  "oracle_layer_rows", "oracle_router_affinity", "oracle_layer_rows_ex",
                  "oracle_layer_rows_mt",
                  "oracle_hash_route", "oracle_bias_update", "oracle_fp8_quantize_row",
                  "oracle_fp8_dequantize_row", "oracle_ep_plan", "oracle_ep_token_plan",
                  "oracle_ep_token_base"):
            getattr(_lib, f).restype = C.c_int
    return _lib


def _np(a, dtype):
    """Host array view with the given numpy dtype (bf16 torch tensors -> uint16 bits)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if a.dtype == torch.bfloat16:
                a = a.view(torch.int16).numpy().view(np.uint16)
            else:
                a = a.numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    if a.dtype != np.dtype(dtype):
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return a


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _check(rc, what):
    if rc != OK:
        raise RuntimeError(f"{what} failed with oracle status {rc}")


AFFINITY_SIGMOID, AFFINITY_SQRT_SOFTPLUS = 0, 1
ROUTER_SIGMOID, ROUTER_SQRT_SOFTPLUS, ROUTER_HASH = 0, 1, 2


def router_scores(x, e, logit_offset=None, rows=None, affinity=AFFINITY_SIGMOID):
    """fp32 affinities f(x[rows] . e_i + o_i), shape [n_rows, E]; f = sigmoid
    (affinity 0) or sqrt(softplus) (affinity 1)."""
    x = _np(x, np.uint16)
    e = _np(e, np.float32)
    off = None if logit_offset is None else _np(logit_offset, np.float32)
    T, d = x.shape
    E = e.shape[0]
    r = None if rows is None else _np(np.asarray(rows, dtype=np.int64), np.int64)
    n = T if r is None else len(r)
    out = np.empty((n, E), np.float32)
    _check(lib().oracle_router_affinity(n, _p(r), d, E, _p(x), _p(e), _p(off), int(affinity),
                                        _p(out)), "oracle_router_affinity")
    return out


def lowbias32(v):
    return int(lib().oracle_lowbias32(C.c_uint32(int(v) & 0xFFFFFFFF)))


def hash_route(token_ids, E, G, K, M):
    """Hash router: returns (topk_idx int32 [n,K], topk_w fp32 [n,K]) for int64 token ids."""
    ids = _np(np.asarray(token_ids, dtype=np.int64), np.int64)
    n = len(ids)
    idx = np.empty((n, K), np.int32)
    w = np.empty((n, K), np.float32)
    _check(lib().oracle_hash_route(n, _p(ids), E, G, K, M, _p(idx), _p(w)), "oracle_hash_route")
    return idx, w


def bias_update(counts, T, K, gamma, bias):
    """Returns bias + gamma * sign(T*K/E - counts) (fp32), the input left as is."""
    c = _np(np.asarray(counts, dtype=np.int32), np.int32)
    b = np.array(_np(bias, np.float32), copy=True)
    _check(lib().oracle_bias_update(len(c), int(T), int(K), _p(c), C.c_float(gamma), _p(b)),
           "oracle_bias_update")
    return b


def select(scores, bias, G, K, M, want_group_score=False):
    """Node-limited top-K: returns (topk_idx int32 [n,K], topk_w fp32 [n,K][, group_score])."""
    s = _np(scores, np.float32)
    b = _np(bias, np.float32)
    n, E = s.shape
    idx = np.empty((n, K), np.int32)
    w = np.empty((n, K), np.float32)
    gs = np.empty((n, G), np.float32) if want_group_score else None
    _check(lib().oracle_select(n, E, G, K, M, _p(s), _p(b), _p(idx), _p(w), _p(gs)),
           "oracle_select")
    return (idx, w, gs) if want_group_score else (idx, w)


def dispatch(topk_idx, E, G):
    """Counting-sort dispatch; returns a dict of int32 arrays."""
    idx = _np(topk_idx, np.int32)
    T, K = idx.shape
    out = {
        "counts": np.empty(E, np.int32), "offsets": np.empty(E + 1, np.int32),
        "send": np.empty((G, G), np.int32), "send_tok": np.empty((G, G), np.int32),
        "perm_token": np.empty(T * K, np.int32), "inv_perm": np.empty((T, K), np.int32),
    }
    rc = lib().oracle_dispatch(T, E, G, K, _p(idx), _p(out["counts"]), _p(out["offsets"]),
                               _p(out["send"]), _p(out["send_tok"]), _p(out["perm_token"]),
                               _p(out["inv_perm"]))
    if rc != OK:
        raise ValueError(f"oracle_dispatch rejected the routing (status {rc})")
    return out


def ffn_row(x_row, Wg, Wu, Wd, round_h=False):
    x_row = _np(x_row, np.uint16)
    Wg, Wu, Wd = _np(Wg, np.uint16), _np(Wu, np.uint16), _np(Wd, np.uint16)
    d_ff, d = Wg.shape
    y = np.empty(d, np.float64)
    _check(lib().oracle_ffn_row(d, d_ff, _p(x_row), _p(Wg), _p(Wu), _p(Wd), int(round_h), _p(y)),
           "oracle_ffn_row")
    return y


def shared_row(x_row, Wsg, Wsu, Wsd, round_h=False):
    x_row = _np(x_row, np.uint16)
    Wsg, Wsu, Wsd = _np(Wsg, np.uint16), _np(Wsu, np.uint16), _np(Wsd, np.uint16)
    ns, ffs, d = Wsg.shape
    y = np.empty(d, np.float64)
    _check(lib().oracle_shared_row(d, ns, ffs, _p(x_row), _p(Wsg), _p(Wsu), _p(Wsd),
                                   int(round_h), _p(y)), "oracle_shared_row")
    return y


def combine(y_perm, inv_perm, topk_w, y_shared=None):
    yp = _np(y_perm, np.uint16)
    ip = _np(inv_perm, np.int32)
    w = _np(topk_w, np.float32)
    ys = None if y_shared is None else _np(y_shared, np.uint16)
    T, K = ip.shape
    d = yp.shape[1]
    out = np.empty((T, d), np.float64)
    _check(lib().oracle_combine(T, d, K, yp.shape[0], _p(yp), _p(ip), _p(w), _p(ys), _p(out)),
           "oracle_combine")
    return out


def e4m3_decode(code):
    return float(lib().oracle_e4m3_decode(int(code) & 0xFF))


def e4m3_encode(v):
    return int(lib().oracle_e4m3_encode(C.c_float(float(v))))


def ep_plan(counts_all):
    """Expert-parallel row placement from counts_all [world, E]: returns
    (base [world, E], local_offsets [world, E/world + 1]) int32."""
    c = _np(np.asarray(counts_all, dtype=np.int32), np.int32)
    world, E = c.shape
    base = np.empty((world, E), np.int32)
    loff = np.empty((world, E // world + 1), np.int32)
    _check(lib().oracle_ep_plan(world, E, _p(c), _p(base), _p(loff)), "oracle_ep_plan")
    return base, loff


def ep_token_plan(topk_idx, E, world):
    """Deduplicated dispatch of one rank: (tok_slot [T, world], tok_counts
    [world]) int32; tok_slot -1 where a token has no expert at that owner."""
    idx = _np(np.asarray(topk_idx, dtype=np.int32), np.int32)
    T, K = idx.shape
    slot = np.empty((T, world), np.int32)
    cnt = np.empty(world, np.int32)
    _check(lib().oracle_ep_token_plan(T, K, E, world, _p(idx), _p(slot), _p(cnt)),
           "oracle_ep_token_plan")
    return slot, cnt


def ep_token_base(tok_counts_all):
    """tok_base [world, world] from tok_counts_all [world, world] (row r = rank
    r's per-owner token counts): first row of rank r's tokens at owner o."""
    c = _np(np.asarray(tok_counts_all, dtype=np.int32), np.int32)
    world = c.shape[0]
    base = np.empty((world, world), np.int32)
    _check(lib().oracle_ep_token_base(world, _p(c), _p(base)), "oracle_ep_token_base")
    return base


def fp8_quantize(x):
    """FP8 payload of bf16 rows x [n, d]: (q uint8 [n, d], scale fp32 [n, d/128])."""
    x = _np(x, np.uint16)
    x2 = x.reshape(-1, x.shape[-1])
    n, d = x2.shape
    q = np.empty((n, d), np.uint8)
    sc = np.empty((n, d // 128), np.float32)
    for r in range(n):
        _check(lib().oracle_fp8_quantize_row(d, _p(x2[r]), _p(q[r]), _p(sc[r])),
               "oracle_fp8_quantize_row")
    return q.reshape(x.shape), sc.reshape(x.shape[:-1] + (d // 128,))


def fp8_dequantize(q, scale):
    """bf16 bits (uint16) the expert GEMM sees for an FP8 payload."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sc = np.ascontiguousarray(scale, dtype=np.float32)
    q2 = q.reshape(-1, q.shape[-1])
    s2 = sc.reshape(-1, sc.shape[-1])
    out = np.empty(q2.shape, np.uint16)
    for r in range(q2.shape[0]):
        _check(lib().oracle_fp8_dequantize_row(q2.shape[1], _p(q2[r]), _p(s2[r]), _p(out[r])),
               "oracle_fp8_dequantize_row")
    return out.reshape(q.shape)


def layer_rows(rows, shape, x, router_w, bias, w_gate, w_up, w_down, ws_gate, ws_up, ws_down,
               logit_offset=None, round_h=False, router=ROUTER_SIGMOID, token_ids=None,
               payload=0, threads=1):
    """The whole layer for the token rows ``rows``.

    ``w_gate``/``w_up``/``w_down`` are sequences of per-expert host matrices
    (entries may be None for experts no listed token selects).
    ``router`` is ROUTER_SIGMOID, ROUTER_SQRT_SOFTPLUS or ROUTER_HASH (the
    last keyed by ``token_ids[row]``, or the row index when None); ``payload``
    1 feeds the routed experts the FP8 round trip of x.  ``threads`` > 1 runs
    the same per-row definition on that many contiguous row shards in parallel
    POSIX threads (``all_cores()`` = every host core); the result is the same.
    Returns (out float64 [n,d], topk_idx [n,K], topk_w [n,K], scores [n,E]).
    """
    r = _np(np.asarray(rows, dtype=np.int64), np.int64)
    x = _np(x, np.uint16)
    e = None if router_w is None else _np(router_w, np.float32)
    b = None if bias is None else _np(bias, np.float32)
    off = None if logit_offset is None else _np(logit_offset, np.float32)
    tid = None if token_ids is None else _np(np.asarray(token_ids, dtype=np.int64), np.int64)
    keep = []

    def parr(mats):
        arr = (C.c_void_p * shape.E)()
        for i, m in enumerate(mats):
            if m is not None:
                a = _np(m, np.uint16)
                keep.append(a)
                arr[i] = a.ctypes.data
        return arr

    g, u, dn = parr(w_gate), parr(w_up), parr(w_down)
    sg, su, sd = (_np(ws_gate, np.uint16), _np(ws_up, np.uint16), _np(ws_down, np.uint16))
    n = len(r)
    out = np.empty((n, shape.d), np.float64)
    idx = np.empty((n, shape.K), np.int32)
    w = np.empty((n, shape.K), np.float32)
    sc = np.empty((n, shape.E), np.float32)
    sc.fill(np.nan)
    rc = lib().oracle_layer_rows_mt(int(threads), n, _p(r), shape.d, shape.E, shape.G, shape.K,
                                    shape.M,
                                    shape.d_ff, shape.n_shared, shape.d_ff_shared,
                                    _p(x), _p(e), _p(off), _p(b), int(router), _p(tid),
                                    int(payload),
                                    C.cast(g, C.c_void_p), C.cast(u, C.c_void_p),
                                    C.cast(dn, C.c_void_p), _p(sg), _p(su), _p(sd),
                                    int(round_h), _p(out), _p(idx), _p(w), _p(sc))
    _check(rc, "oracle_layer_rows_mt")
    return out, idx, w, sc


def all_cores() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):  # pragma: no cover
        return os.cpu_count() or 1
