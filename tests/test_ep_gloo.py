"""Host side of the expert-parallel step with real process groups (gloo,
world size 2, CPU): every rank gathers the per-expert counts of all ranks in
rank order, and the row placement each rank derives from them matches the one
derived from the whole batch in one process; with the deduplicated
dispatch the per-owner token counts travel in the same exchange."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _worker(rank, world, port, E, K, T, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import sys
        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        from combine_expert_ffn_b200.ep import gather_counts
        import oracle
        rng = np.random.default_rng(42)
        idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
        Tr = T // world
        mine = np.bincount(idx[rank * Tr:(rank + 1) * Tr].ravel(), minlength=E).astype(np.int32)
        slot, tok = oracle.ep_token_plan(idx[rank * Tr:(rank + 1) * Tr], E, world)
        # one exchange of the per-expert copy counts and the per-owner token counts
        got = gather_counts(torch.from_numpy(np.concatenate([mine, tok]))).numpy()
        counts_all, tok_counts_all = got[:, :E], got[:, E:]
        base, loff = oracle.ep_plan(counts_all)
        tok_base = oracle.ep_token_base(tok_counts_all)
        q.put((rank, counts_all.tolist(), base[rank].tolist(), loff[rank].tolist(),
               tok_base[rank].tolist()))
    finally:
        dist.destroy_process_group()


def test_counts_exchange_and_plan_with_two_ranks(orc):
    pytest.importorskip("torch.distributed")
    E, K, T, world = 16, 4, 64, 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, world, port, E, K, T, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict()
    for _ in range(world):
        rank, counts_all, base, loff, tok_base = q.get(timeout=120)
        got[rank] = (counts_all, base, loff, tok_base)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    rng = np.random.default_rng(42)
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    Tr = T // world
    counts_all = np.stack([np.bincount(idx[r * Tr:(r + 1) * Tr].ravel(), minlength=E)
                           for r in range(world)])
    base, loff = orc.ep_plan(counts_all)
    tok_counts_all = np.stack([orc.ep_token_plan(idx[r * Tr:(r + 1) * Tr], E, world)[1]
                               for r in range(world)])
    tok_base = orc.ep_token_base(tok_counts_all)
    for r in range(world):
        assert got[r][0] == counts_all.tolist()
        assert got[r][1] == base[r].tolist()
        assert got[r][2] == loff[r].tolist()
        assert got[r][3] == tok_base[r].tolist()
