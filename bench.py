#!/usr/bin/env python
"""Throughput of the MoE layer forward on B200 (tokens/s), with rooflines.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config v3] [--impl ours|reference]

One step = one whole layer forward (route -> dispatch -> expert FFN ->
combine) over one batch of seeded synthetic tokens of the named workload,
inputs resident in HBM.  The stages are issued as the four ABI calls that
moe_forward makes, with CUDA events between them on the launching stream, so
the timed region also yields each stage's device time.  `e2e` times the
public moe_forward call on pinned HOST buffers with every step's host->device
copy of x and device->host copy of the output inside the timed region, the
copies of neighbouring steps overlapping the compute as in a serving loop.

Multi-GPU: the layer does not shard (one GPU per layer instance), so N > 1
runs N independent replicas, one per rank, each on its own batch; the job's
value is all ranks' tokens / the slowest rank's time.

`--impl reference` times the CPU oracle, as it stands, on the host cores over a
bounded sample of tokens of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s on 1 B200; grouped-GEMM % bf16 peak; permute/combine % HBM"
UNIT = "tokens/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# fp32 CUDA-core peak for the router logits: 148 SMs x 128 FMA lanes x 2 FLOP x clock
FP32_LANES = 148 * 128 * 2


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(PEAKS_FALLBACK)
    d["source"] = "fallback"
    return d


def algorithmic(sh):
    """Per-token algorithmic work of each stage (bytes or FLOPs)."""
    T, d, E, K, ff = sh.T, sh.d, sh.E, sh.K, sh.d_ff
    shared_ff = sh.n_shared * sh.d_ff_shared
    return {
        # route: read x row (bf16) + write K idx/w; router weights read once per batch
        "route_flop": 2.0 * E * d,
        # dispatch: read x once, write K copies (bf16) + 3 int32 index words per copy
        "dispatch_bytes": 2.0 * d * (1 + K) + 4.0 * 3 * K,
        # its gather-permute part: read x once, read K row indices, write K copies
        "permute_bytes": 2.0 * d * (1 + K) + 4.0 * K,
        # expert FFN: 6 d d_ff per token-expert (gate, up, down), routed + shared
        "ffn_flop": 6.0 * d * (ff * K + shared_ff),
        # combine: read K y rows + y_shared + K (idx, w), write out
        "combine_bytes": 2.0 * d * (K + 2) + 8.0 * K,
    }


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("gemm_sm100.cu", "common.cuh"):
        with open(os.path.join(ROOT, "combine_expert_ffn_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def traffic_from_profile(sh):
    """DRAM bytes per step of the expert FFN (both GEMM launches) from the committed
    ncu summary, if it was taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "expert_ffn_traffic.txt")
    if not os.path.exists(p):
        return None
    d = {}
    with open(p) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            k, v = line.split(":", 1)
            d[k.strip()] = v.strip()
    if d.get("source_sha256") != kernel_source_hash() or d.get("workload") != sh.name:
        return None
    return int(d["dram_bytes_per_step"])


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "samples": len(sm),
                "reasons": sorted(reasons)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world, device="cuda"):
    """The slowest rank's time (every rank gets the same value)."""
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank, world, steps, ms_max):
    """Whole-job throughput: every replica's tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (ms_max / 1e3)


# ---------------------------------------------------------------- CPU oracle
def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class OracleHost:
    """Host copies of one workload's inputs for the CPU oracle.

    The routed experts' weights are copied from the device once, as the sampled
    tokens first need them, and reused by later samples."""

    def __init__(self, sh, inp):
        import oracle
        oracle.build()
        self.oracle, self.sh, self.inp = oracle, sh, inp
        self.x, self.e, self.b = inp["x"].cpu(), inp["router_w"].cpu(), inp["bias"].cpu()
        off = inp.get("logit_offset")
        self.off = off.cpu() if off is not None else None
        self.g, self.u, self.d = [None] * sh.E, [None] * sh.E, [None] * sh.E
        self.sg, self.su, self.sd = (inp["ws_gate"].cpu(), inp["ws_up"].cpu(),
                                     inp["ws_down"].cpu())

    def tokens_per_s(self, n_tokens, seed_offset=0, threads=1):
        """Times the oracle's whole layer on `n_tokens` spread tokens over `threads`
        host threads; returns (tokens/s, seconds)."""
        import numpy as np
        sh, orc = self.sh, self.oracle
        rows = (np.linspace(0, sh.T - 1, n_tokens).astype(np.int64) + seed_offset) % sh.T
        scores = orc.router_scores(self.x, self.e, self.off, rows=rows)
        idx, _ = orc.select(scores, self.b, sh.G, sh.K, sh.M)
        for ex in sorted(set(int(v) for v in idx.ravel())):
            if self.g[ex] is None:
                self.g[ex] = self.inp["w_gate"][ex].cpu()
                self.u[ex] = self.inp["w_up"][ex].cpu()
                self.d[ex] = self.inp["w_down"][ex].cpu()
        t0 = time.perf_counter()
        orc.layer_rows(rows, sh, self.x, self.e, self.b, self.g, self.u, self.d, self.sg,
                       self.su, self.sd, logit_offset=self.off, threads=threads)
        dt = time.perf_counter() - t0
        return n_tokens / dt, dt


def cpu_baseline_leg(args, sh, inp):
    """The oracle as it stands on this machine's host cores: one thread over
    `--cpu-tokens` tokens, then every core over `--cpu-tokens-per-core` tokens
    per core (a bounded sample of the same workload, the tokens spread over the
    batch).  The all-core rate is the reported value."""
    import oracle
    host = OracleHost(sh, inp)
    cores = oracle.all_cores()
    v1, dt1 = host.tokens_per_s(args.cpu_tokens, threads=1)
    n_all = max(args.cpu_tokens, args.cpu_tokens_per_core * cores)
    va, dta = host.tokens_per_s(n_all, seed_offset=1, threads=cores)
    return {
        "value": va, "unit": UNIT, "cores": cores, "kind": "oracle",
        "sample": f"{n_all} tokens of the {sh.name} workload spread over the batch, whole layer "
                  f"per token (routing, {sh.K} routed + {sh.n_shared} shared SwiGLU FFNs, combine), "
                  f"{cores} threads, {dta:.1f} s",
        "nproc": os.cpu_count(), "cpu_model": cpu_model(),
        "single_core": {"value": v1, "unit": UNIT, "cores": 1,
                        "sample": f"{args.cpu_tokens} tokens, one thread, {dt1:.1f} s"},
        "all_core": {"value": va, "unit": UNIT, "cores": cores,
                     "sample": f"{n_all} tokens, {cores} threads, {dta:.1f} s"},
    }


def run_reference(args, sh, world, rank):
    if rank != 0:
        return 0
    import oracle
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = synth.make_inputs(sh, dev)
    host = OracleHost(sh, inp)
    cores = oracle.all_cores()
    n = args.ref_tokens_per_core * cores
    vals, total = [], 0.0
    for i in range(args.warmup + args.steps):
        v, dt = host.tokens_per_s(n, seed_offset=i, threads=cores)
        if i >= args.warmup:
            vals.append(v)
            total += dt
    value = n * args.steps / total
    sample = (f"{n} tokens per step of the {sh.name} workload (routing + {sh.K} routed + "
              f"{sh.n_shared} shared SwiGLU FFN per token), {cores} threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded counter-based generator)",
        "config": {"workload": sh.name, **sh.as_dict(), "tokens_per_step": n},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample, "nproc": os.cpu_count(), "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- ours
def run_ours(args, sh, world, rank, local):
    import combine_expert_ffn_b200 as moe

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    sh_rank = sh.replace(seed=sh.seed) if world == 1 else sh
    inp = synth.make_inputs(sh_rank, dev)
    if world > 1 and rank > 0:   # replicas: each rank its own batch of tokens
        inp["x"] = synth.normal(sh.seed + 1000 * rank, synth.TENSOR_IDS["x"], (sh.T, sh.d),
                                sh.x_sigma, torch.bfloat16, dev)
    cfg = moe.MoeConfig.of(sh)
    ws = moe.alloc_workspace(cfg, dev)
    o = moe.forward_outputs(cfg, dev)
    T, K, E, G, d = sh.T, sh.K, sh.E, sh.G, sh.d
    # expert weights in the library's tile-packed layout: transformed once here, at
    # load time, outside every timed region (the row-major copies stay for the e2e
    # leg's reference and are not read by the packed path)
    packed = None
    if args.weights == "packed":
        packed = moe.pack_weights(cfg, inp["w_gate"], inp["w_up"], inp["w_down"],
                                  inp["ws_gate"], inp["ws_up"], inp["ws_down"], device=dev)
        torch.cuda.synchronize(dev)
    # stage buffers (the same intermediates moe_forward keeps in its workspace)
    perm_token = torch.empty(T * K, dtype=torch.int32, device=dev)
    inv_perm = torch.empty(T, K, dtype=torch.int32, device=dev)
    y_perm = torch.empty(T * K, d, dtype=torch.bfloat16, device=dev)
    y_sh = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    x_perm = torch.empty(T * K, d, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        moe.moe_route(cfg, inp["x"], inp["router_w"], inp.get("logit_offset"), inp["bias"],
                      o["topk_idx"], o["topk_w"], None, ws, stream)
        if ev is not None:
            ev[1].record(stream)
        # the dispatch as its two parts: the plan (counting sort of the copies), then
        # the gather-permute of the x rows (together: moe_dispatch with x_perm)
        moe.moe_dispatch(cfg, inp["x"], o["topk_idx"], o["counts"], o["offsets"], o["send"],
                         o["send_tok"], perm_token, inv_perm, None, ws, stream)
        if ev is not None:
            ev[2].record(stream)
        moe.moe_permute(cfg, inp["x"], inv_perm, x_perm, stream)
        if ev is not None:
            ev[3].record(stream)
        if packed is not None:
            moe.moe_expert_ffn_packed(cfg, x_perm, o["offsets"], packed, y_perm, inp["x"], y_sh,
                                      ws, stream)
        else:
            moe.moe_expert_ffn(cfg, x_perm, o["offsets"], inp["w_gate"], inp["w_up"],
                               inp["w_down"], y_perm, inp["x"], inp["ws_gate"], inp["ws_up"],
                               inp["ws_down"], y_sh, ws, stream)
        if ev is not None:
            ev[4].record(stream)
        moe.moe_combine(cfg, y_perm, inv_perm, o["topk_w"], y_sh, o["out"], stream)
        if ev is not None:
            ev[5].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if moe.moe_read_device_status(ws) != moe.MOE_OK:
        raise RuntimeError("device status after warm-up: %d" % moe.moe_read_device_status(ws))

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.25)  # let the sampler take its first sample
    n0 = moe.moe_launch_count()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    launches = moe.moe_launch_count() - n0
    clk = clocks.stop()
    barrier(world)
    ms_total = max_over_ranks(start.elapsed_time(end), world)
    stage_ms = {k: 0.0 for k in ("route", "dispatch_plan", "permute", "expert_ffn", "combine")}
    for ev in evs:
        for j, k in enumerate(stage_ms):
            stage_ms[k] += ev[j].elapsed_time(ev[j + 1])
    stage_ms = {k: v / args.steps for k, v in stage_ms.items()}
    stage_ms["dispatch"] = stage_ms["dispatch_plan"] + stage_ms["permute"]
    # per-step device times (first stage event to last), for the median and minimum
    step_ms = [ev[0].elapsed_time(ev[5]) for ev in evs]
    status = moe.moe_read_device_status(ws)
    if status != moe.MOE_OK:
        raise RuntimeError(f"device status {status} after the timed region")

    # ---- end to end through moe_forward with pinned host buffers
    e2e = e2e_leg(args, sh, cfg, inp, ws, o, stream, dev, world, packed) \
        if not args.no_e2e else None
    if rank != 0:
        return 0
    counts = o["counts"].cpu()
    line = report(args, sh, world, ms_total, stage_ms, launches, clk, e2e,
                  touched_experts=int((counts > 0).sum()), step_ms=step_ms)
    # the routing of the timed batch: expert loads and the group-to-group send matrices
    line["routing"] = {
        "max_over_mean_expert_load": float(counts.max()) / (T * K / E),
        "min_over_mean_expert_load": float(counts.min()) / (T * K / E),
        "send": o["send"].cpu().tolist(),
        "send_tok": o["send_tok"].cpu().tolist(),
    }
    if not args.no_variants:
        line["variants"] = variants_leg(sh, inp, dev, stream)
    if args.ep_world > 1:
        line["expert_parallel"] = ep_leg(sh, inp, dev, stream, args.ep_world)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_leg(args, sh, inp)
    print(json.dumps(line), flush=True)
    return 0


def e2e_leg(args, sh, cfg, inp, ws, o, stream, dev, world, packed=None):
    """moe_forward on pinned host buffers, every step's H2D of x and D2H of out
    inside the timed region.  Steps are pipelined the way a serving loop runs
    them: x of step i+1 goes up on a copy stream and out of step i-1 comes
    down on another while step i computes (two device buffers each; events
    order every reuse)."""
    import combine_expert_ffn_b200 as moe
    T, d = sh.T, sh.d
    NB = 2
    x_host = inp["x"].cpu().pin_memory()
    out_host = [torch.empty(T, d, dtype=torch.bfloat16).pin_memory() for _ in range(NB)]
    x_dev = [torch.empty_like(inp["x"]) for _ in range(NB)]
    out_dev = [torch.empty(T, d, dtype=torch.bfloat16, device=dev) for _ in range(NB)]
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    up_done = [torch.cuda.Event() for _ in range(NB)]
    fwd_done = [torch.cuda.Event() for _ in range(NB)]
    down_done = [torch.cuda.Event() for _ in range(NB)]

    def run(n):
        for i in range(n):
            b = i % NB
            if i >= NB:
                s_up.wait_event(fwd_done[b])       # step i-NB has read x_dev[b]
            with torch.cuda.stream(s_up):
                x_dev[b].copy_(x_host, non_blocking=True)
            up_done[b].record(s_up)
            stream.wait_event(up_done[b])
            if i >= NB:
                stream.wait_event(down_done[b])    # step i-NB's out_dev[b] is on the host
            if packed is not None:
                moe.moe_forward_packed(cfg, x_dev[b], inp["router_w"], inp.get("logit_offset"),
                                       inp["bias"], packed, out_dev[b], ws=ws, stream=stream)
            else:
                moe.moe_forward(cfg, x_dev[b], inp["router_w"], inp.get("logit_offset"),
                                inp["bias"], inp["w_gate"], inp["w_up"], inp["w_down"],
                                inp["ws_gate"], inp["ws_up"], inp["ws_down"], out_dev[b], ws=ws,
                                stream=stream)
            fwd_done[b].record(stream)
            s_down.wait_event(fwd_done[b])
            with torch.cuda.stream(s_down):
                out_host[b].copy_(out_dev[b], non_blocking=True)
            down_done[b].record(s_down)

    run(args.warmup)
    barrier(world)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    run(args.steps)
    e1.record(s_down)                              # after the last step's D2H
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = job_tokens_per_s(T, world, args.steps, e2e_ms)
    if not torch.equal(out_host[(args.steps - 1) % NB], o["out"].cpu()) and world == 1:
        raise RuntimeError("moe_forward and the staged calls disagree")
    return {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": T * d * 2,
            "d2h_bytes_per_step": T * d * 2, "pipelined": "H2D, forward and D2H of consecutive steps on three streams"}


def variants_leg(sh, inp, dev, stream, reps=20):
    """Device times of the routing variants and the bias update (CUDA events,
    mean over `reps` back-to-back launches after 3 warm-ups): the route stage
    under each router, moe_forward under each router, and moe_bias_update.
    Not part of the headline step."""
    import combine_expert_ffn_b200 as moe
    T, K, E = sh.T, sh.K, sh.E
    ids = synth.token_ids(sh.seed, T, device=dev)
    idx = torch.empty(T, K, dtype=torch.int32, device=dev)
    w = torch.empty(T, K, dtype=torch.float32, device=dev)
    bias = inp["bias"].clone()

    def timed(fn):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / reps

    out = {}
    # the dispatch gather fused into the expert FFN vs the two-step path
    cfg = moe.MoeConfig.of(sh)
    ws = moe.alloc_workspace(cfg, dev)
    o = moe.forward_outputs(cfg, dev)
    perm = torch.empty(T * K, dtype=torch.int32, device=dev)
    inv = torch.empty(T, K, dtype=torch.int32, device=dev)
    x_perm = torch.empty(T * K, sh.d, dtype=torch.bfloat16, device=dev)
    y_perm = torch.empty(T * K, sh.d, dtype=torch.bfloat16, device=dev)
    y_sh = torch.empty(T, sh.d, dtype=torch.bfloat16, device=dev)
    moe.moe_route(cfg, inp["x"], inp["router_w"], inp.get("logit_offset"), inp["bias"],
                  o["topk_idx"], o["topk_w"], None, ws, stream)

    def two_step():
        moe.moe_dispatch(cfg, inp["x"], o["topk_idx"], o["counts"], o["offsets"], o["send"],
                         o["send_tok"], perm, inv, x_perm, ws, stream)
        moe.moe_expert_ffn(cfg, x_perm, o["offsets"], inp["w_gate"], inp["w_up"], inp["w_down"],
                           y_perm, inp["x"], inp.get("ws_gate"), inp.get("ws_up"),
                           inp.get("ws_down"), y_sh, ws, stream)

    def fused():
        moe.moe_dispatch(cfg, inp["x"], o["topk_idx"], o["counts"], o["offsets"], o["send"],
                         o["send_tok"], perm, inv, None, ws, stream)
        moe.moe_expert_ffn_gather(cfg, inp["x"], perm, o["offsets"], inp["w_gate"], inp["w_up"],
                                  inp["w_down"], y_perm, inp.get("ws_gate"), inp.get("ws_up"),
                                  inp.get("ws_down"), y_sh, ws, stream)

    res = {"two_step_x_perm": timed(two_step), "fused_gather": timed(fused)}
    if sh.d % 128 == 0:  # the FP8 payload: 1-byte codes + 1x128 scales
        cfg8 = moe.MoeConfig.of(sh, payload=moe.MOE_PAYLOAD_FP8)
        xq = torch.empty(T * K, sh.d, dtype=torch.uint8, device=dev)
        xs = torch.empty(T * K, sh.d // 128, dtype=torch.float32, device=dev)

        def fp8_payload():
            moe.moe_dispatch_fp8(cfg8, inp["x"], o["topk_idx"], o["counts"], o["offsets"],
                                 o["send"], o["send_tok"], perm, inv, xq, xs, ws, stream)
            moe.moe_expert_ffn_fp8(cfg8, xq, xs, o["offsets"], inp["w_gate"], inp["w_up"],
                                   inp["w_down"], y_perm, inp["x"], inp.get("ws_gate"),
                                   inp.get("ws_up"), inp.get("ws_down"), y_sh, ws, stream)

        res["fp8_payload"] = timed(fp8_payload)
        del xq, xs
    out["dispatch_plus_ffn_ms"] = res
    # moe_forward replayed from a CUDA graph (launch overheads gone)
    g = torch.cuda.CUDAGraph()
    s_cap = torch.cuda.Stream(dev)
    s_cap.wait_stream(stream)
    with torch.cuda.stream(s_cap):
        with torch.cuda.graph(g, stream=s_cap):
            moe.moe_forward(cfg, inp["x"], inp["router_w"], inp.get("logit_offset"), inp["bias"],
                            inp["w_gate"], inp["w_up"], inp["w_down"], inp.get("ws_gate"),
                            inp.get("ws_up"), inp.get("ws_down"), o["out"], ws=ws, stream=s_cap)
    stream.wait_stream(s_cap)
    gms = timed(g.replay)
    out["graph_forward"] = {"forward_ms": gms, "forward_tokens_per_s": T / (gms / 1e3)}
    del g
    del ws, o, x_perm, y_perm, y_sh
    if sh.d % 128 == 0:
        cfg8 = moe.MoeConfig.of(sh, payload=moe.MOE_PAYLOAD_FP8)
        ws8 = moe.alloc_workspace(cfg8, dev)
        o8 = moe.forward_outputs(cfg8, dev)
        ms = timed(lambda: moe.moe_forward(cfg8, inp["x"], inp["router_w"],
                                           inp.get("logit_offset"), inp["bias"], inp["w_gate"],
                                           inp["w_up"], inp["w_down"], inp.get("ws_gate"),
                                           inp.get("ws_up"), inp.get("ws_down"), o8["out"],
                                           ws=ws8, stream=stream))
        out["fp8_payload_forward"] = {"forward_ms": ms, "forward_tokens_per_s": T / (ms / 1e3)}
        del ws8, o8
    names = {moe.MOE_ROUTER_SIGMOID: "sigmoid", moe.MOE_ROUTER_SQRT_SOFTPLUS: "sqrt_softplus",
             moe.MOE_ROUTER_HASH: "hash"}
    for r, name in names.items():
        cfg = moe.MoeConfig.of(sh, router=r)
        ws = moe.alloc_workspace(cfg, dev)
        o = moe.forward_outputs(cfg, dev)
        if r == moe.MOE_ROUTER_HASH:
            route = lambda: moe.moe_route_hash(cfg, ids, idx, w, stream)  # noqa: E731
        else:
            route = lambda: moe.moe_route(cfg, inp["x"], inp["router_w"],  # noqa: E731
                                          inp.get("logit_offset"), inp["bias"], idx, w, None,
                                          ws, stream)
        fwd = lambda: moe.moe_forward(cfg, inp["x"], inp["router_w"],  # noqa: E731
                                      inp.get("logit_offset"), inp["bias"], inp["w_gate"],
                                      inp["w_up"], inp["w_down"], inp.get("ws_gate"),
                                      inp.get("ws_up"), inp.get("ws_down"), o["out"],
                                      counts=o["counts"], ws=ws, stream=stream, token_ids=ids)
        route_ms, fwd_ms = timed(route), timed(fwd)
        if moe.moe_read_device_status(ws, stream) != moe.MOE_OK:
            raise RuntimeError(f"device status after the {name} router variant")
        out[name] = {"route_ms": route_ms, "forward_ms": fwd_ms,
                     "forward_tokens_per_s": T / (fwd_ms / 1e3)}
        if r == moe.MOE_ROUTER_SIGMOID:
            out["bias_update_ms"] = timed(lambda: moe.moe_bias_update(cfg, o["counts"], 1e-3,
                                                                      bias, stream))
        del ws, o
    return out


# measured peer copy over NVLink 5, one direction per GPU (GB/s)
NVLINK_GBS = 770.0


def ep_leg(sh, inp, dev, stream, world, reps=20):
    """Expert parallelism over `world` ranks, emulated on this GPU: every rank
    of the step runs in sequence with same-device pointer tables (peer stores
    and loads become local HBM traffic).  Reports each stage's device time
    (every rank's launches of the stage replayed from one CUDA graph) summed
    over the ranks and per rank, the fused dispatch and combine
    against the HBM peak, and the bytes of those two exchanges that would
    cross NVLink on `world` GPUs with their time at the measured peer-copy
    bandwidth (the larger of a rank's outgoing and incoming bytes).  Not part
    of the headline step."""
    import combine_expert_ffn_b200 as moe
    from combine_expert_ffn_b200 import ep
    if sh.T % world or sh.E % world or (sh.T // world) % sh.G:
        return {"world": world, "skipped": "T, E or T/world not divisible"}
    em = ep.EmulatedEP(sh, inp, world, stream=stream)
    em.forward()
    torch.cuda.synchronize(dev)
    for st in em.ranks:
        if int(st.status.item()) != moe.MOE_OK or moe.moe_read_device_status(st.ws) != moe.MOE_OK:
            raise RuntimeError("device status after the emulated EP step")

    def timed(fn):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / reps

    def graphed(stage):
        # one stage of all ranks captured once and replayed: the host's
        # per-call overhead would otherwise exceed the short kernels' time
        g = torch.cuda.CUDAGraph()
        s_cap = torch.cuda.Stream(dev)
        s_cap.wait_stream(stream)
        em.stream = s_cap
        with torch.cuda.stream(s_cap):
            with torch.cuda.graph(g, stream=s_cap):
                getattr(em, stage)()
        em.stream = stream
        stream.wait_stream(s_cap)
        return g

    stages = ("route_and_plan_local", "exchange_counts", "plan", "dispatch", "expert_ffn",
              "combine")
    graphs = {k: graphed(k) for k in stages}
    # the HBM-bound exchange stages first, the expert GEMMs (which pull the SM
    # clock down to the power cap) last
    timing_order = ("exchange_counts", "plan", "dispatch", "combine", "route_and_plan_local",
                    "expert_ffn")
    t_ms = {k: timed(graphs[k].replay) for k in timing_order}
    all_ranks = {k: t_ms[k] for k in stages}
    for st in em.ranks:
        if int(st.status.item()) != moe.MOE_OK or moe.moe_read_device_status(st.ws) != moe.MOE_OK:
            raise RuntimeError("device status after the emulated EP stages")
    del graphs
    Tr, d, K, E = sh.T // world, sh.d, sh.K, sh.E
    El = E // world
    hbm = load_peaks()["hbm_gbs"]
    disp_bytes = (2.0 * d * (1 + K) + 8.0 * K) * Tr      # x row, K copies, idx + inv
    comb_bytes = (2.0 * d * (K + 1 + (1 if sh.n_shared else 0)) + 12.0 * K) * Tr
    per_rank = {k: v / world for k, v in all_ranks.items()}
    ca = em.counts_all.cpu().to(torch.int64)
    owner = torch.arange(E) // El
    out_copies = [int(ca[r][owner != r].sum()) for r in range(world)]
    in_copies = [int(ca[:, owner == o].sum() - ca[o, owner == o].sum()) for o in range(world)]
    link_bytes = 2.0 * d * max(max(out_copies), max(in_copies))
    res = {
        "world": world, "tokens_per_rank": Tr,
        "stage_ms_all_ranks": all_ranks, "stage_ms_per_rank": per_rank,
        "dispatch": {"bytes_per_rank": disp_bytes,
                     "achieved_gbs": disp_bytes / (per_rank["dispatch"] / 1e3) / 1e9,
                     "frac_of_hbm": disp_bytes / (per_rank["dispatch"] / 1e3) / 1e9 / hbm},
        "combine": {"bytes_per_rank": comb_bytes,
                    "achieved_gbs": comb_bytes / (per_rank["combine"] / 1e3) / 1e9,
                    "frac_of_hbm": comb_bytes / (per_rank["combine"] / 1e3) / 1e9 / hbm},
        "nvlink": {"max_rank_bytes_per_exchange": link_bytes,
                   "projected_ms_per_exchange": link_bytes / (NVLINK_GBS * 1e9) * 1e3,
                   "bandwidth_gbs": NVLINK_GBS, "copies_out": out_copies, "copies_in": in_copies},
        "note": "all ranks run in sequence on one GPU; peer traffic is local HBM here",
    }
    del em
    # the deduplicated dispatch: each token crosses once to each owner holding
    # one of its experts, plus a 4-byte fan-out index per copy; the owner
    # rebuilds its copy rows locally
    torch.cuda.empty_cache()
    em = ep.EmulatedEP(sh, inp, world, stream=stream, dedup=True, dedup_combine=True)
    em.forward()
    torch.cuda.synchronize(dev)
    dd_stages = ("dispatch", "fanout", "precombine", "combine")
    graphs = {k: graphed(k) for k in dd_stages}
    td = {k: timed(graphs[k].replay) / world for k in dd_stages}
    for st in em.ranks:
        if int(st.status.item()) != moe.MOE_OK or moe.moe_read_device_status(st.ws) != moe.MOE_OK:
            raise RuntimeError("device status after the emulated deduplicated dispatch")
    del graphs
    tca = em.gathered[:, E:].cpu().to(torch.int64)              # [world, world] tokens
    tok_out = [int(tca[r].sum() - tca[r, r]) for r in range(world)]
    tok_in = [int(tca[:, o].sum() - tca[o, o]) for o in range(world)]
    dd_link = 2.0 * d * max(max(tok_out), max(tok_in)) + 4.0 * max(max(out_copies),
                                                                  max(in_copies))
    mean_tok_rows = float(tca.sum()) / world
    dd_bytes = 2.0 * d * (Tr + mean_tok_rows) + 12.0 * K * Tr   # x read, token rows, indices
    fan_bytes = 4.0 * d * (Tr * K) + 4.0 * Tr * K               # copy rows read + written
    dd_comb_link = 2.0 * d * max(max(tok_out), max(tok_in))     # one partial row per pair
    res["dedup_dispatch"] = {
        "stage_ms_per_rank": td,
        "token_rows_per_rank": mean_tok_rows,
        "dispatch": {"bytes_per_rank": dd_bytes,
                     "achieved_gbs": dd_bytes / (td["dispatch"] / 1e3) / 1e9,
                     "frac_of_hbm": dd_bytes / (td["dispatch"] / 1e3) / 1e9 / hbm},
        "fanout": {"bytes_per_rank": fan_bytes,
                   "achieved_gbs": fan_bytes / (td["fanout"] / 1e3) / 1e9,
                   "frac_of_hbm": fan_bytes / (td["fanout"] / 1e3) / 1e9 / hbm},
        "nvlink": {"max_rank_bytes_dispatch": dd_link,
                   "projected_ms_dispatch": dd_link / (NVLINK_GBS * 1e9) * 1e3,
                   "max_rank_bytes_combine": dd_comb_link,
                   "projected_ms_combine": dd_comb_link / (NVLINK_GBS * 1e9) * 1e3,
                   "tokens_out": tok_out, "tokens_in": tok_in},
        "note": "dispatch stage includes the combine's list plan; combine = one partial row "
                "per (token, owner), summed by the owner (precombine) before the exchange",
    }
    del em
    if sh.d % 128 == 0:
        # the FP8 payload: E4M3 codes + one fp32 scale per 128 channels travel
        # instead of bf16 rows; the owners' GEMM widens them
        torch.cuda.empty_cache()
        em = ep.EmulatedEP(sh, inp, world, stream=stream, payload=moe.MOE_PAYLOAD_FP8)
        em.forward()
        torch.cuda.synchronize(dev)
        graphs = {k: graphed(k) for k in ("dispatch", "expert_ffn")}
        t8 = {k: timed(graphs[k].replay) / world for k in ("dispatch", "expert_ffn")}
        for st in em.ranks:
            if int(st.status.item()) != moe.MOE_OK or \
                    moe.moe_read_device_status(st.ws) != moe.MOE_OK:
                raise RuntimeError("device status after the emulated FP8 EP stages")
        del graphs
        q_bytes = (2.0 * d + K * (d + d / 32.0) + 8.0 * K) * Tr   # x read, codes + scales
        q_link = (d + d / 32.0) * max(max(out_copies), max(in_copies))
        del em
        torch.cuda.empty_cache()
        # ... and sent once per (token, owner), fanned out at the owner
        em = ep.EmulatedEP(sh, inp, world, stream=stream, payload=moe.MOE_PAYLOAD_FP8,
                           dedup=True)
        em.forward()
        torch.cuda.synchronize(dev)
        graphs = {k: graphed(k) for k in ("dispatch", "fanout")}
        t8d = {k: timed(graphs[k].replay) / world for k in ("dispatch", "fanout")}
        for st in em.ranks:
            if int(st.status.item()) != moe.MOE_OK:
                raise RuntimeError("device status after the emulated FP8 deduplicated dispatch")
        del graphs
        q_dd_link = (d + d / 32.0) * max(max(tok_out), max(tok_in)) + \
            4.0 * max(max(out_copies), max(in_copies))
        res["fp8_payload"] = {
            "dedup": {"stage_ms_per_rank": t8d,
                      "nvlink": {"max_rank_bytes_dispatch": q_dd_link,
                                 "projected_ms_dispatch": q_dd_link / (NVLINK_GBS * 1e9) * 1e3}},
            "stage_ms_per_rank": t8,
            "dispatch": {"bytes_per_rank": q_bytes,
                         "achieved_gbs": q_bytes / (t8["dispatch"] / 1e3) / 1e9,
                         "frac_of_hbm": q_bytes / (t8["dispatch"] / 1e3) / 1e9 / hbm},
            "nvlink": {"max_rank_bytes_dispatch": q_link,
                       "projected_ms_dispatch": q_link / (NVLINK_GBS * 1e9) * 1e3},
        }
        del em
    return res


def report(args, sh, world, ms_total, stage_ms, launches, clk, e2e, touched_experts=None,
           step_ms=None):
    T = sh.T
    ms_step = ms_total / args.steps
    step_ms = step_ms or [ms_step]
    value = job_tokens_per_s(T, world, args.steps, ms_total)
    peaks = load_peaks()
    alg = algorithmic(sh)
    ffn_s = stage_ms["expert_ffn"] / 1e3
    ffn_tflops = alg["ffn_flop"] * T / ffn_s / 1e12
    # the timed region is a fraction of a second of short steps: the burst peak applies
    tensor_peak = peaks["bf16_tflops"]
    hbm = peaks["hbm_gbs"]
    clock_for_alu = (clk or {}).get("sm_mhz") or peaks.get("sm_max_mhz", 1965.0)
    route_tflops = alg["route_flop"] * T / (stage_ms["route"] / 1e3) / 1e12
    fp32_peak = FP32_LANES * clock_for_alu * 1e6 / 1e12
    disp_gbs = alg["dispatch_bytes"] * T / (stage_ms["dispatch"] / 1e3) / 1e9
    perm_gbs = alg["permute_bytes"] * T / (stage_ms["permute"] / 1e3) / 1e9
    comb_gbs = alg["combine_bytes"] * T / (stage_ms["combine"] / 1e3) / 1e9
    traffic = traffic_from_profile(sh)
    # expert weights the step reads: every routed expert that got a row, plus the shared ones
    touched = sh.E if touched_experts is None else touched_experts
    w_bytes = 2.0 * 3 * sh.d * (touched * sh.d_ff + sh.n_shared * sh.d_ff_shared)
    w_gbs = w_bytes / ffn_s / 1e9
    # below the ridge (FLOPs per weight byte < tensor peak / HBM bandwidth) the expert FFN is
    # bound by streaming its weights, and that is the roofline reported
    weight_bound = alg["ffn_flop"] * T / w_bytes < tensor_peak * 1e12 / (hbm * 1e9)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded counter-based generator, random-init weights)",
        "config": {"workload": sh.name, **sh.as_dict(), "parallelism": f"replicas x{world}",
                   "expert_weights": (
                       "tile-packed (moe_pack_weights, once at load, outside the timed region)"
                       if args.weights == "packed" else "row-major"),
                   "l2": "inputs larger than L2: %.1f GB of expert weights streamed per step"
                         % ((3 * sh.E * sh.d * sh.d_ff + 3 * sh.n_shared * sh.d * sh.d_ff_shared) * 2 / 1e9)},
        "roofline": ({"bound": "tensor", "kernel": "expert FFN: grouped_ffn_gemm_kernel<SwiGLU> + <store> (2 launches)",
                      "achieved": ffn_tflops, "peak": tensor_peak, "unit": "TFLOP/s",
                      "frac": ffn_tflops / tensor_peak,
                      "peak_kind": f"{peaks['source']} bf16 burst",
                      "frac_of_sustained": ffn_tflops / peaks.get("bf16_tflops_sustained",
                                                                  peaks["bf16_tflops"]),
                      "traffic": traffic}
                     if not weight_bound else
                     {"bound": "hbm", "kernel": "expert FFN: grouped_ffn_gemm_kernel<SwiGLU> + <store> (2 launches)",
                      "achieved": w_gbs, "peak": hbm, "unit": "GB/s", "frac": w_gbs / hbm,
                      "peak_kind": f"{peaks['source']} HBM copy",
                      "basis": "bytes of the expert weights touched (%d of %d routed experts + shared) per launch pair"
                               % (touched, sh.E),
                      "tensor_tflops": ffn_tflops, "traffic": traffic}),
        "expert_weights": {"touched_experts": touched, "bytes": w_bytes, "achieved_gbs": w_gbs,
                           "frac_of_hbm": w_gbs / hbm},
        "stages": {
            "ms": stage_ms,
            "route": {"bound": "tensor", "achieved": route_tflops, "unit": "TFLOP/s",
                      "peak": peaks["bf16_tflops"], "frac": route_tflops / peaks["bf16_tflops"],
                      "note": "algorithmic 2*E*d per token; the kernel issues 3 bf16 MMAs per "
                              "product (fp32 weights split into exact bf16 parts); "
                              "fp32 CUDA-core peak at the sampled clock: %.1f TFLOP/s" % fp32_peak},
            "dispatch": {"bound": "hbm", "achieved": disp_gbs, "unit": "GB/s", "peak": hbm,
                         "frac": disp_gbs / hbm, "note": "plan + permute"},
            "permute": {"bound": "hbm", "achieved": perm_gbs, "unit": "GB/s", "peak": hbm,
                        "frac": perm_gbs / hbm},
            "combine": {"bound": "hbm", "achieved": comb_gbs, "unit": "GB/s", "peak": hbm,
                        "frac": comb_gbs / hbm},
        },
        "gpu_launches": int(launches),
        "e2e": e2e,
        "clocks": clk,
    }
    line["ms_per_step_median"] = statistics.median(step_ms)
    line["ms_per_step_min"] = min(step_ms)
    # a compact copy of the per-stage times and fractions next to the dominant kernel's line
    st = line["stages"]
    line["roofline"]["step_ms"] = {"mean": ms_step, "median": line["ms_per_step_median"],
                                   "min": line["ms_per_step_min"]}
    line["roofline"]["other_stages"] = {
        "route": {"ms": stage_ms["route"], "tflops": route_tflops,
                  "frac_of_bf16_peak": st["route"]["frac"]},
        "dispatch": {"ms": stage_ms["dispatch"], "gbs": disp_gbs, "frac_of_hbm": disp_gbs / hbm},
        "permute": {"ms": stage_ms["permute"], "gbs": perm_gbs, "frac_of_hbm": perm_gbs / hbm},
        "combine": {"ms": stage_ms["combine"], "gbs": comb_gbs, "frac_of_hbm": comb_gbs / hbm},
        "hbm_peak_gbs": hbm, "peaks": peaks["source"],
    }
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="v3", choices=sorted(synth.CONFIGS) + sorted(synth.PROFILE_CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=24,
                    help="tokens of the single-thread oracle sample")
    ap.add_argument("--cpu-tokens-per-core", type=int, default=8,
                    help="tokens per host core of the all-core oracle sample")
    ap.add_argument("--ref-tokens-per-core", type=int, default=1,
                    help="tokens per host core in each step of the reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg (profiling runs)")
    ap.add_argument("--ep-world", type=int, default=8,
                    help="ranks of the emulated expert-parallel leg (1 = skip)")
    ap.add_argument("--weights", default="packed", choices=["packed", "row-major"],
                    help="expert weights in the tile-packed layout (packed once at load) or "
                         "row-major")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the router-variant and bias-update timings")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    sh = synth.config(args.config)
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            return run_reference(args, sh, world, rank)
        return run_ours(args, sh, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
