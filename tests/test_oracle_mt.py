"""The all-core oracle driver runs the single-threaded definition on row shards.

Rows of the layer never interact, so splitting the token rows over threads
must give exactly the bytes of one single-threaded call: outputs, routing,
gates and affinities.  Checked on the ragged workload (several shards, a
shard count that does not divide the rows, more threads than rows) for the
sigmoid, sqrt(softplus) and hash routers and the FP8 payload.
"""
import numpy as np
import pytest

import synth
from tests import harness as H


def _run(orc, sh, inp, rows, threads, router=0, payload=0):
    tid = np.arange(sh.T, dtype=np.int64) * 7 + 3 if router == 2 else None
    return orc.layer_rows(rows, sh, inp["x"], inp["router_w"], inp["bias"],
                          list(inp["w_gate"]), list(inp["w_up"]), list(inp["w_down"]),
                          inp["ws_gate"], inp["ws_up"], inp["ws_down"], router=router,
                          token_ids=tid, payload=payload, threads=threads)


@pytest.mark.parametrize("router,payload", [(0, 0), (1, 0), (2, 0), (0, 1)])
def test_threaded_oracle_equals_single_thread(orc, router, payload):
    # the FP8 payload needs d % 128 == 0
    sh = H.RAGGED if payload == 0 else H.RAGGED.replace(name="ragged_d256", d=256)
    inp = synth.make_inputs(sh, "cpu")
    rows = np.arange(0, sh.T, 3, dtype=np.int64)  # 88 rows, not a multiple of 3 or 5
    ref = _run(orc, sh, inp, rows, 1, router, payload)
    for threads in (2, 3, 5, len(rows) + 4):
        got = _run(orc, sh, inp, rows, threads, router, payload)
        for a, b in zip(ref, got):
            if a.dtype.kind == "f":
                np.testing.assert_array_equal(a.view(np.uint8), b.view(np.uint8))
            else:
                np.testing.assert_array_equal(a, b)


def test_all_cores_is_positive(orc):
    assert orc.all_cores() >= 1


def test_parity_rows_pick_the_heavy_tails_and_high_rows(orc):
    """The full-size parity sampler's row map is the oracle dispatch's, and it
    picks tokens in the most-loaded experts' last tiles and the highest rows."""
    sh = synth.config("skew").replace(name="skew_small", T=20480, d=7168)
    rng = np.random.default_rng(3)
    gsz = sh.E // sh.G
    idx = np.empty((sh.T, sh.K), np.int32)
    for t in range(sh.T):  # K distinct experts in M groups, skewed towards group 0
        groups = rng.choice(sh.G, sh.M, replace=False, p=np.r_[0.5, np.full(sh.G - 1, 0.5 / (sh.G - 1))])
        idx[t] = np.concatenate([g * gsz + rng.choice(gsz, sh.K // sh.M, replace=False)
                                 for g in groups])
    ref = orc.dispatch(idx, sh.E, sh.G)
    rows = H.copy_rows(idx, sh.E)
    np.testing.assert_array_equal(rows, ref["inv_perm"])
    pick = H.parity_rows(sh, idx, n_spread=64)
    assert len(pick) >= 64 and np.all(np.diff(pick) > 0)
    counts = ref["counts"]
    heavy = int(np.argmax(counts))
    last_tile = (counts[heavy] - 1) // 128 * 128
    seg_tokens = ref["perm_token"][ref["offsets"][heavy] + last_tile:ref["offsets"][heavy + 1]]
    assert set(seg_tokens.tolist()) & set(pick.tolist())
    top = int(rows.max())
    assert np.any(rows[pick] == top)
    # 20480 * 8 rows of 14336 bytes pass the 2^31-byte offset: rows just past it are picked
    first_high = -(-(2 ** 31) // (2 * sh.d))
    assert np.any((rows[pick] >= first_high) & (rows[pick] < first_high + 24))
