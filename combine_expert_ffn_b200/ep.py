"""Expert parallelism over ranks: the host-side steps around the EP entry
points of libmoe (argument marshalling and the collectives that order them).

A rank owns E / world experts and routes its own tokens.  One step:

    moe_route, moe_dispatch(x_perm=None)     local routing and dispatch plan
      (+ moe_ep_token_plan, dedup)            tokens per owner
    all-gather of the per-expert counts       counts_all [world, E]
      (+ the per-owner token counts)
    moe_ep_plan (+ moe_ep_token_base)         where this rank's copies go
    moe_ep_dispatch                           gather + peer stores (bf16 rows, or
                                              E4M3 codes + scales: moe_ep_dispatch_fp8;
                                              or one row per token and owner plus a
                                              fan-out index per copy: dedup)
      (+ moe_ep_combine_plan, dedup_combine)  copy rows and gates per token, owner
                                              (bf16 dedup: moe_ep_dispatch_dedup_plan,
                                              one launch for both)
    barrier                                   every rank's stores are done
    (moe_ep_fanout, dedup)                    the owner's copy rows from token rows
    moe_ep_expert_ffn                         this rank's experts, shared experts
    (moe_ep_precombine, dedup_combine)        one partial row per token, owner
    barrier                                   every rank's outputs are done
    moe_ep_combine                            peer loads + gate-weighted sum
      (moe_ep_combine_dedup)                  or one partial row per owner

`EPLayer` runs that step in a process group of one process per GPU, with the
receive buffers mapped into every rank by CUDA IPC and the barriers as
stream-ordered all-reduces.  `emulate_forward` runs all ranks of one step on a
single GPU, one after the other (no rank waits on another inside a kernel),
with the same kernels and plain same-device pointers in the tables.
"""
from __future__ import annotations

import torch

from . import (MoeConfig, moe_dispatch, moe_ep_combine, moe_ep_combine_dedup,
               moe_ep_combine_plan, moe_ep_dispatch, moe_ep_dispatch_dedup,
               moe_ep_dispatch_dedup_fp8, moe_ep_dispatch_dedup_plan, moe_ep_dispatch_fp8,
               moe_ep_expert_ffn, moe_ep_expert_ffn_fp8, moe_ep_fanout, moe_ep_fanout_fp8,
               moe_ep_plan, moe_ep_precombine, moe_ep_token_base, moe_ep_token_plan,
               moe_ep_workspace_size, moe_ipc_close_handle, moe_ipc_get_handle,
               moe_ipc_open_handle, moe_route, moe_route_hash, MOE_PAYLOAD_FP8, MOE_ROUTER_HASH)


def _i32(n, device):
    return torch.empty(n, dtype=torch.int32, device=device)


class _RankState:
    """Per-rank buffers of one EP step."""

    # bf16 dedup with the deduplicated combine: dispatch and combine lists in one
    # launch (moe_ep_dispatch_dedup_plan); False: the two separate launches
    fused_plan = True

    def __init__(self, cfg: MoeConfig, world: int, device, dedup: bool = False,
                 dedup_combine: bool = False):
        T, K, E, G, d = cfg.T, cfg.K, cfg.E, cfg.G, cfg.d
        if dedup_combine and not dedup:
            raise ValueError("the deduplicated combine runs on the deduplicated dispatch")
        self.cfg, self.world, self.dedup, self.dedup_combine = cfg, world, dedup, dedup_combine
        self.topk_idx = torch.empty(T, K, dtype=torch.int32, device=device)
        self.topk_w = torch.empty(T, K, dtype=torch.float32, device=device)
        self.counts, self.offsets = _i32(E, device), _i32(E + 1, device)
        self.send = torch.empty(G, G, dtype=torch.int32, device=device)
        self.send_tok = torch.empty(G, G, dtype=torch.int32, device=device)
        self.perm, self.inv = _i32(T * K, device), torch.empty(T, K, dtype=torch.int32, device=device)
        self.base, self.local_offsets = _i32(E, device), _i32(E // world + 1, device)
        cap = world * T * K
        self.fp8 = cfg.payload == MOE_PAYLOAD_FP8
        if dedup:      # one row per (token, owner); the owner fans out locally
            if self.fp8:   # codes + scales per token row
                self.recv_tq = torch.empty(world * T, d, dtype=torch.uint8, device=device)
                self.recv_ts = torch.empty(world * T, d // 128, dtype=torch.float32,
                                           device=device)
            else:
                self.recv_tok = torch.empty(world * T, d, dtype=torch.bfloat16, device=device)
            self.recv_idx = torch.empty(cap, dtype=torch.int32, device=device)
            self.tok_slot = torch.empty(T, world, dtype=torch.int32, device=device)
            self.tok_counts, self.tok_base = _i32(world, device), _i32(world + 1, device)
        if dedup_combine:  # per (token, owner): copy rows + gates; one partial row back
            self.recv_list = _i32(world * T * K, device)
            self.recv_lw = torch.empty(world * T * K, dtype=torch.float32, device=device)
            self.recv_lcnt = _i32(world * T, device)
            self.partial = torch.empty(world * T, d, dtype=torch.bfloat16, device=device)
        if self.fp8:   # E4M3 codes + one fp32 scale per 128 channels
            self.recv_x = None
            self.recv_q = torch.empty(cap, d, dtype=torch.uint8, device=device)
            self.recv_scale = torch.empty(cap, d // 128, dtype=torch.float32, device=device)
        else:
            self.recv_x = torch.empty(cap, d, dtype=torch.bfloat16, device=device)
        self.recv_y = torch.empty(cap, d, dtype=torch.bfloat16, device=device)
        self.y_shared = torch.empty(T, d, dtype=torch.bfloat16, device=device)
        self.out = torch.empty(T, d, dtype=torch.bfloat16, device=device)
        n = moe_ep_workspace_size(cfg, world)
        self.ws = torch.empty(n, dtype=torch.uint8, device=device)
        self.ws[:256].zero_()
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def route_and_plan_local(self, x, router_w, logit_offset, bias, token_ids, stream):
        cfg = self.cfg
        if cfg.router == MOE_ROUTER_HASH:
            moe_route_hash(cfg, token_ids, self.topk_idx, self.topk_w, stream)
        else:
            moe_route(cfg, x, router_w, logit_offset, bias, self.topk_idx, self.topk_w, None,
                      self.ws, stream)
        moe_dispatch(cfg, x, self.topk_idx, self.counts, self.offsets, self.send, self.send_tok,
                     self.perm, self.inv, None, self.ws, stream)
        if self.dedup:
            moe_ep_token_plan(cfg, self.world, self.topk_idx, self.tok_slot, self.tok_counts,
                              stream)

    def exchanged(self):
        """What every rank sends in the all-gather: the per-expert copy counts
        (and, deduplicating, the per-owner token counts), one int32 vector."""
        return torch.cat([self.counts, self.tok_counts]) if self.dedup else self.counts

    def plan(self, world, rank, gathered, stream):
        """gathered [world, len(exchanged())]: every rank's exchanged vector."""
        E = self.cfg.E
        moe_ep_plan(self.cfg, world, rank, gathered[:, :E].contiguous(), self.base,
                    self.local_offsets, stream)
        if self.dedup:
            moe_ep_token_base(self.cfg, world, rank, gathered[:, E:].contiguous(), self.tok_base,
                              stream)

    def recv_buffers(self):
        """The buffers the dispatch writes into at this rank as an owner."""
        if self.dedup:
            extra = [self.recv_list, self.recv_lw, self.recv_lcnt] if self.dedup_combine else []
            rows = [self.recv_tq, self.recv_ts] if self.fp8 else [self.recv_tok]
            return rows + [self.recv_idx] + extra
        return [self.recv_q, self.recv_scale] if self.fp8 else [self.recv_x]

    def combine_buffer(self):
        """The buffer the other ranks' combines read at this rank."""
        return self.partial if self.dedup_combine else self.recv_y

    def precombine(self, stream):
        """Deduplicated combine: this owner's partial rows."""
        if self.dedup_combine:
            moe_ep_precombine(self.cfg, self.world, self.recv_y, self.recv_list, self.recv_lw,
                              self.recv_lcnt, self.tok_base, self.partial, self.status, stream)

    def combine(self, world, table, stream):
        """table: device pointer table of the ranks' combine_buffer()."""
        y_sh = self.y_shared if self.cfg.n_shared else None
        if self.dedup_combine:
            moe_ep_combine_dedup(self.cfg, world, self.topk_idx, self.tok_slot, self.tok_base,
                                 table, y_sh, self.out, self.status, stream)
        else:
            moe_ep_combine(self.cfg, world, self.topk_idx, self.topk_w, self.offsets, self.inv,
                           self.base, table, y_sh, self.out, self.status, stream)

    def fanout(self, stream):
        """Deduplicating: this owner's copy rows from its token rows."""
        if self.dedup and self.fp8:
            moe_ep_fanout_fp8(self.cfg, self.world, self.recv_tq, self.recv_ts, self.recv_idx,
                              self.local_offsets, self.recv_q, self.recv_scale, self.status,
                              stream)
        elif self.dedup:
            moe_ep_fanout(self.cfg, self.world, self.recv_tok, self.recv_idx, self.local_offsets,
                          self.recv_x, self.status, stream)

    def dispatch(self, world, x, tables, stream):
        """tables: one device pointer table per entry of recv_buffers()."""
        if self.dedup:
            if self.fp8:
                moe_ep_dispatch_dedup_fp8(self.cfg, world, x, self.topk_idx, self.offsets,
                                          self.inv, self.base, self.tok_slot, self.tok_base,
                                          tables[0], tables[1], tables[2], self.status, stream)
                lists = tables[3:]
            elif self.dedup_combine and self.fused_plan:  # the lists from the same launch
                moe_ep_dispatch_dedup_plan(self.cfg, world, x, self.topk_idx, self.topk_w,
                                           self.offsets, self.inv, self.base, self.tok_slot,
                                           self.tok_base, tables[0], tables[1], tables[2],
                                           tables[3], tables[4], self.status, stream)
                return
            else:
                moe_ep_dispatch_dedup(self.cfg, world, x, self.topk_idx, self.offsets, self.inv,
                                      self.base, self.tok_slot, self.tok_base, tables[0],
                                      tables[1], self.status, stream)
                lists = tables[2:]
            if self.dedup_combine:
                moe_ep_combine_plan(self.cfg, world, self.topk_idx, self.topk_w, self.offsets,
                                    self.inv, self.base, self.tok_slot, self.tok_base, lists[0],
                                    lists[1], lists[2], self.status, stream)
        elif self.fp8:
            moe_ep_dispatch_fp8(self.cfg, world, x, self.topk_idx, self.offsets, self.inv,
                                self.base, tables[0], tables[1], self.status, stream)
        else:
            moe_ep_dispatch(self.cfg, world, x, self.topk_idx, self.offsets, self.inv, self.base,
                            tables[0], self.status, stream)

    def expert_ffn(self, world, rank, w, x, w_shared, stream):
        y_sh = self.y_shared if self.cfg.n_shared else None
        if self.fp8:
            moe_ep_expert_ffn_fp8(self.cfg, world, rank, self.recv_q, self.recv_scale,
                                  self.local_offsets, *w, self.recv_y, x, *w_shared, y_sh,
                                  self.ws, stream)
        else:
            moe_ep_expert_ffn(self.cfg, world, rank, self.recv_x, self.local_offsets, *w,
                              self.recv_y, x, *w_shared, y_sh, self.ws, stream)


def gather_counts(counts, group=None):
    """counts_all [world, E]: every rank's per-expert copy counts, in rank order."""
    import torch.distributed as dist
    parts = [torch.empty_like(counts) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, counts, group=group)
    return torch.stack(parts)


def _local_weights(w, rank, world):
    El = w.shape[0] // world
    return w[rank * El:(rank + 1) * El]


class EmulatedEP:
    """All `world` ranks of one EP step on this GPU.  The batch is split into
    equal contiguous chunks (T % world == 0 and (T / world) % G == 0).  Each
    stage method runs that stage for every rank in rank order; a stage starts
    only after the previous one has run for all ranks, which stands in for the
    barriers between them."""

    def __init__(self, shape, inp: dict, world: int, router=None, token_ids=None, stream=None,
                 payload=None, dedup=False, dedup_combine=False):
        self.device = inp["x"].device
        base_cfg = MoeConfig.of(shape, router=router)
        T = base_cfg.T
        if T % world or base_cfg.E % world:
            raise ValueError("T and E must be multiples of world")
        Tr = T // world
        self.world, self.stream, self.inp = world, stream, inp
        self.cfg = MoeConfig.of(shape.replace(T=Tr), router=router, payload=payload)
        self.ranks = [_RankState(self.cfg, world, self.device, dedup, dedup_combine)
                      for _ in range(world)]
        self.xs = [inp["x"][r * Tr:(r + 1) * Tr] for r in range(world)]
        self.ids = [None if token_ids is None else token_ids[r * Tr:(r + 1) * Tr]
                    for r in range(world)]
        n_buf = len(self.ranks[0].recv_buffers())
        self.recv_tables = [torch.tensor([st.recv_buffers()[i].data_ptr() for st in self.ranks],
                                         dtype=torch.int64, device=self.device)
                            for i in range(n_buf)]
        self.recv_y_ptrs = torch.tensor([st.combine_buffer().data_ptr() for st in self.ranks],
                                        dtype=torch.int64, device=self.device)
        n_ex = self.ranks[0].exchanged().numel()
        self.gathered = torch.empty(world, n_ex, dtype=torch.int32, device=self.device)

    def route_and_plan_local(self):
        inp = self.inp
        for r, st in enumerate(self.ranks):
            st.route_and_plan_local(self.xs[r], inp["router_w"], inp.get("logit_offset"),
                                    inp["bias"], self.ids[r], self.stream)

    @property
    def counts_all(self):
        return self.gathered[:, :self.cfg.E]

    def exchange_counts(self):
        # the all-gather: row r is rank r's exchanged vector
        with torch.cuda.stream(self.stream or torch.cuda.current_stream(self.device)):
            for r, st in enumerate(self.ranks):
                self.gathered[r].copy_(st.exchanged())

    def plan(self):
        for r, st in enumerate(self.ranks):
            st.plan(self.world, r, self.gathered, self.stream)

    def dispatch(self):
        for r, st in enumerate(self.ranks):
            st.dispatch(self.world, self.xs[r], self.recv_tables, self.stream)

    def fanout(self):
        for st in self.ranks:
            st.fanout(self.stream)

    def expert_ffn(self):
        inp, world = self.inp, self.world
        w_shared = (inp.get("ws_gate"), inp.get("ws_up"), inp.get("ws_down"))
        for r, st in enumerate(self.ranks):
            w = tuple(_local_weights(inp[k], r, world) for k in ("w_gate", "w_up", "w_down"))
            st.expert_ffn(world, r, w, self.xs[r], w_shared, self.stream)

    def precombine(self):
        for st in self.ranks:
            st.precombine(self.stream)

    def combine(self):
        for st in self.ranks:
            st.combine(self.world, self.recv_y_ptrs, self.stream)

    def forward(self):
        self.route_and_plan_local()
        self.exchange_counts()
        self.plan()
        self.dispatch()
        self.fanout()
        self.expert_ffn()
        self.precombine()
        self.combine()
        return torch.cat([st.out for st in self.ranks])


def emulate_forward(shape, inp: dict, world: int, router=None, token_ids=None, stream=None,
                    payload=None, dedup=False, dedup_combine=False):
    """One EP step of all `world` ranks on this GPU; returns (out [T, d],
    per-rank states)."""
    em = EmulatedEP(shape, inp, world, router, token_ids, stream, payload, dedup, dedup_combine)
    return em.forward(), em.ranks


class EPLayer:
    """One rank of an expert-parallel MoE layer in a process group with one
    process per GPU.  Holds this rank's experts (w_gate / w_up / w_down
    [E/world, ...]), the replicated router and shared experts, and the receive
    buffers, mapped into every rank by CUDA IPC.

    With the NCCL backend the counts exchange and the barriers are
    stream-ordered collectives (no host synchronisation inside the step);
    call torch.cuda.set_device for this rank's GPU before constructing it.
    With gloo they run on the host after synchronising the step's stream;
    that form also lets several processes share one GPU (each maps the
    others' buffers through IPC on the same device).
    """

    def __init__(self, shape_local, group, router_w, bias, w_gate_local, w_up_local,
                 w_down_local, ws_gate=None, ws_up=None, ws_down=None, logit_offset=None,
                 router=None, payload=None, dedup=False, dedup_combine=False):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.device = w_gate_local.device
        self.host_sync = dist.get_backend(group) != "nccl"
        self.cfg = MoeConfig.of(shape_local, router=router, payload=payload)
        self.st = _RankState(self.cfg, self.world, self.device, dedup, dedup_combine)
        self.router_w, self.bias, self.logit_offset = router_w, bias, logit_offset
        self.w = (w_gate_local, w_up_local, w_down_local)
        self.ws_shared = (ws_gate, ws_up, ws_down)
        self._opened = []
        torch.cuda.synchronize(self.device)   # buffers allocated before peers map them
        self.recv_tables = [self._map_peers(b) for b in self.st.recv_buffers()]
        self.recv_y_ptrs = self._map_peers(self.st.combine_buffer())
        self._flag = torch.zeros(1, dtype=torch.int32, device=self.device)

    def _map_peers(self, buf):
        handles = [None] * self.world
        self.dist.all_gather_object(handles, moe_ipc_get_handle(buf), group=self.group)
        ptrs = []
        for r, h in enumerate(handles):
            if r == self.rank:
                ptrs.append(buf.data_ptr())
            else:
                p = moe_ipc_open_handle(h)
                self._opened.append(p)
                ptrs.append(p)
        return torch.tensor(ptrs, dtype=torch.int64, device=self.device)

    def _barrier(self, stream):
        """Every rank's work issued so far on its step stream has completed
        before any rank's later work on that stream starts."""
        if self.host_sync:
            stream.synchronize()
            self.dist.barrier(group=self.group)
        else:
            self.dist.all_reduce(self._flag, group=self.group)

    def _gather(self, counts, stream):
        if self.host_sync:
            stream.synchronize()
            return gather_counts(counts.cpu(), self.group).to(self.device)
        return gather_counts(counts, self.group)

    def forward(self, x, token_ids=None, stream=None):
        """This rank's tokens x [T, d] -> out [T, d] (a buffer of the layer,
        overwritten by the next call)."""
        st, cfg, world, r = self.st, self.cfg, self.world, self.rank
        s = stream or torch.cuda.current_stream(self.device)
        with torch.cuda.stream(s):   # the collectives order against this stream
            st.route_and_plan_local(x, self.router_w, self.logit_offset, self.bias, token_ids, s)
            st.plan(world, r, self._gather(st.exchanged(), s), s)
            self._barrier(s)          # every rank's receive buffers are free again
            st.dispatch(world, x, self.recv_tables, s)
            self._barrier(s)          # every copy has landed
            st.fanout(s)
            st.expert_ffn(world, r, self.w, x, self.ws_shared, s)
            st.precombine(s)
            self._barrier(s)          # every expert output is written
            st.combine(world, self.recv_y_ptrs, s)
        return st.out

    def close(self, stream=None):
        """Unmaps the peers' buffers once every rank has finished reading
        them (a barrier first); every rank calls it."""
        s = stream or torch.cuda.current_stream(self.device)
        with torch.cuda.stream(s):
            self._barrier(s)
        s.synchronize()
        for p in self._opened:
            moe_ipc_close_handle(p)
        self._opened = []
