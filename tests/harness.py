"""Shared helpers of the parity tests: workloads, oracle sampling, comparisons.

Test infrastructure: imports the oracle and the CUDA binding side by side;
nothing in the product imports this module.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import synth

# Tolerances of the layer (see the test docstrings for where they come from).
TOL_AFFINITY = 1e-5      # |s_gpu - s_oracle|, absolute
TOL_FROB = 5e-3          # ||out_gpu - out_ref||_F / ||out_ref||_F
TOL_ELEM = 2e-2          # max |out_gpu - out_ref| / max |out_ref|

# Small workloads the oracle finishes in seconds that still span several GEMM
# tiles and ragged tails: 320 = 5 k-blocks, d_ff 192 = 1.5 column tiles of the
# gate/up GEMM, d 320 = 1.25 column tiles of the down GEMM, ~88 rows per
# expert with some segments above 128 rows.
RAGGED = synth.MoeShape("ragged", T=264, d=320, E=12, G=4, K=4, M=2, d_ff=192, n_shared=1,
                        d_ff_shared=128, x_sigma=1.0, e_sigma=1 / math.sqrt(320),
                        bias_sigma=0.1, seed=5)
RAGGED2 = synth.MoeShape("ragged2", T=520, d=192, E=40, G=8, K=6, M=3, d_ff=128, n_shared=2,
                         d_ff_shared=64, x_sigma=1 / math.sqrt(192), e_sigma=0.05,
                         bias_sigma=0.05, seed=6)
NOSHARED = synth.MoeShape("noshared", T=96, d=256, E=16, G=4, K=4, M=2, d_ff=128, n_shared=0,
                          d_ff_shared=0, x_sigma=1.0, e_sigma=1 / 16, bias_sigma=0.2, seed=7)
SHAPES = {s.name: s for s in (RAGGED, RAGGED2, NOSHARED)}
SHAPES.update(synth.CONFIGS)


def shape(name: str) -> synth.MoeShape:
    return SHAPES[name]


def host(t):
    return None if t is None else t.detach().cpu()


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def compare_out(gpu_bf16: torch.Tensor, ref: np.ndarray):
    """(relative Frobenius error, max |err| / max |ref|) of bf16 GPU rows vs float64 reference."""
    g = bf16_to_f64(gpu_bf16)
    err = g - ref
    frob = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300))
    elem = float(np.abs(err).max() / max(np.abs(ref).max(), 1e-300))
    return frob, elem


def expert_mats_host(inp: dict, experts, E: int):
    """Per-expert host copies of the routed weights (only the listed experts)."""
    g, u, d = [None] * E, [None] * E, [None] * E
    for e in sorted(set(int(v) for v in experts)):
        g[e] = inp["w_gate"][e].cpu()
        u[e] = inp["w_up"][e].cpu()
        d[e] = inp["w_down"][e].cpu()
    return g, u, d


def copy_rows(topk_idx: np.ndarray, E: int) -> np.ndarray:
    """x_perm row of every copy (t, j) by the stable counting sort's definition:
    expert segments in expert order, tokens ascending inside a segment."""
    T, K = topk_idx.shape
    flat = topk_idx.ravel().astype(np.int64)
    order = np.argsort(flat * (T * K) + np.arange(T * K), kind="stable")
    rows = np.empty(T * K, np.int64)
    rows[order] = np.arange(T * K)
    return rows.reshape(T, K)


def parity_rows(sh: synth.MoeShape, topk_idx: np.ndarray, n_spread: int = 192,
                n_heavy: int = 3, per_tile: int = 12, n_high: int = 24) -> np.ndarray:
    """Token rows for full-size parity, chosen from the routing the GPU produced.

    * ``n_spread`` tokens evenly over the batch;
    * for each of the ``n_heavy`` most-loaded experts, ``per_tile`` tokens whose
      copy is in the expert's last 128-row GEMM tile and ``per_tile`` in the
      tile before it (the longest segments' final tiles);
    * ``n_high`` tokens with a copy at the highest x_perm rows, and, where the
      buffer is longer than 2^31 bytes, ``n_high`` more with a copy just above
      the 2^31-byte offset (64-bit row addressing).
    """
    T, K = topk_idx.shape
    picks = [np.linspace(0, T - 1, min(n_spread, T)).astype(np.int64)]
    rows = copy_rows(topk_idx, sh.E)
    counts = np.bincount(topk_idx.ravel(), minlength=sh.E)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    flat_rows = rows.ravel()
    tok_of_row = np.empty(T * K, np.int64)
    tok_of_row[flat_rows] = np.repeat(np.arange(T), K)
    for e in np.argsort(-counts, kind="stable")[:n_heavy]:
        c = int(counts[e])
        if c == 0:
            continue
        last0 = (c - 1) // 128 * 128
        for lo in (last0, max(0, last0 - 128)):
            seg = np.arange(offsets[e] + lo, offsets[e] + min(c, lo + 128))
            picks.append(tok_of_row[seg[np.linspace(0, len(seg) - 1, min(per_tile, len(seg)))
                                        .astype(np.int64)]])
    picks.append(tok_of_row[T * K - min(n_high, T * K):])
    first_high = -(-(2 ** 31) // (2 * sh.d))  # first row whose byte offset is >= 2^31
    if first_high < T * K:
        picks.append(tok_of_row[first_high:first_high + n_high])
    return np.unique(np.concatenate(picks))


def oracle_layer_sample(orc, sh: synth.MoeShape, inp: dict, rows, router: int = 0,
                        token_ids=None, payload: int = 0, threads: int = 1):
    """Oracle layer output for the token rows `rows` of device inputs `inp`.

    Only the x rows and the experts those tokens choose (by the oracle's own
    routing) are copied to the host.  `router`: 0 sigmoid, 1 sqrt(softplus),
    2 hash keyed by `token_ids` (host int64 [T] or None for the row index);
    `payload` 1 feeds the routed experts the FP8 round trip of x.
    """
    rows = np.asarray(rows, dtype=np.int64)
    x_h = inp["x"].cpu()
    e_h = inp["router_w"].cpu()
    b_h = inp["bias"].cpu()
    off_h = host(inp.get("logit_offset"))
    if router == 2:
        keys = rows if token_ids is None else np.asarray(token_ids, dtype=np.int64)[rows]
        idx, _ = orc.hash_route(keys, sh.E, sh.G, sh.K, sh.M)
    else:
        scores = orc.router_scores(x_h, e_h, off_h, rows=rows, affinity=router)
        idx, _ = orc.select(scores, b_h, sh.G, sh.K, sh.M)
    g, u, d = expert_mats_host(inp, idx.ravel(), sh.E)
    ns = sh.n_shared
    Sg = inp["ws_gate"].cpu() if ns else torch.zeros(1, 64, sh.d, dtype=torch.bfloat16)
    Su = inp["ws_up"].cpu() if ns else torch.zeros(1, 64, sh.d, dtype=torch.bfloat16)
    Sd = inp["ws_down"].cpu() if ns else torch.zeros(1, sh.d, 64, dtype=torch.bfloat16)
    return orc.layer_rows(rows, sh, x_h, e_h, b_h, g, u, d, Sg, Su, Sd, logit_offset=off_h,
                          router=router, token_ids=token_ids, payload=payload, threads=threads)


def near_tie_certified(sh: synth.MoeShape, s_orc: np.ndarray, bias: np.ndarray,
                       idx_gpu, idx_orc, tol: float = TOL_AFFINITY) -> bool:
    """A routing that differs from the oracle's is acceptable only as a near tie.

    With every affinity within `tol` of the oracle's, a correct selector may
    swap two candidates whose oracle-side biased affinities (or group scores)
    differ by at most 2 * tol (2 * K/M * tol for group scores).  All values
    here are the oracle's own.
    """
    E, G, K, M = sh.E, sh.G, sh.K, sh.M
    gsz, kpg = E // G, K // M
    b = (s_orc.astype(np.float64) + bias.astype(np.float64))
    gscore = np.array([np.sort(b[g * gsz:(g + 1) * gsz])[::-1][:kpg].sum() for g in range(G)])
    gs_sorted = np.sort(gscore)[::-1]
    m_th = gs_sorted[M - 1]
    for g in {int(e) // gsz for e in idx_gpu}:
        if gscore[g] < m_th - 2 * kpg * tol:
            return False
    gpu_set, orc_set = set(int(v) for v in idx_gpu), set(int(v) for v in idx_orc)
    if not (gpu_set - orc_set):
        return True
    worst_orc = min(b[e] for e in orc_set)
    return all(b[e] >= worst_orc - 2 * tol for e in gpu_set - orc_set)
