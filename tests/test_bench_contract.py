"""The benchmark's JSON line, built from made-up stage times on the CPU.

Checks the contract's keys and the arithmetic behind them: value = tokens of
all ranks / timed seconds, the roofline fraction = achieved / peak with the
achieved FLOPs from the 6 d d_ff law, HBM fractions from the per-token bytes,
and the DRAM traffic record picked up only for the source it was taken on.
"""
import argparse
import json

import pytest

import bench
import synth

KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "roofline",
        "gpu_launches", "e2e", "clocks", "ms_per_step_median", "ms_per_step_min")


def _line(name="v3", world=1, steps=20, ffn_ms=7.0):
    sh = synth.config(name)
    args = argparse.Namespace(steps=steps, warmup=5, weights="packed")
    stage_ms = {"route": 0.15, "dispatch_plan": 0.03, "permute": 0.2, "expert_ffn": ffn_ms,
                "combine": 0.2}
    stage_ms["dispatch"] = stage_ms["dispatch_plan"] + stage_ms["permute"]
    ms_total = steps * sum(v for k, v in stage_ms.items() if k != "dispatch")
    clk = {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "samples": 3, "reasons": ["sw_power_cap"]}
    e2e = {"value": 1.0, "unit": bench.UNIT, "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 1}
    line = bench.report(args, sh, world, ms_total, stage_ms, 8 * steps, clk, e2e,
                        touched_experts=sh.E, step_ms=[ms_total / steps] * steps)
    return sh, line, ms_total, stage_ms


def test_the_line_has_the_contract_keys_and_is_json():
    _, line, _, _ = _line()
    for k in KEYS:
        assert k in line, k
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in line["roofline"], k
    assert line["config"]["workload"] == "v3" and line["scaling"] == "weak"
    assert line["higher_is_better"] is True and line["dtype"] == "bf16"
    json.loads(json.dumps(line))


@pytest.mark.parametrize("world", [1, 4])
def test_value_counts_every_rank_tokens(world):
    sh, line, ms_total, _ = _line(world=world)
    assert line["value"] == pytest.approx(sh.T * world * 20 / (ms_total / 1e3))
    assert line["ms_per_step"] == pytest.approx(ms_total / 20)


def test_roofline_arithmetic():
    sh, line, _, stage_ms = _line()
    r = line["roofline"]
    flops = 6.0 * sh.d * (sh.K * sh.d_ff + sh.n_shared * sh.d_ff_shared) * sh.T
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(flops / (stage_ms["expert_ffn"] / 1e3) / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    # the combine reads K copies + the shared row and writes out: 2 d (K + 2) + 8 K bytes
    comb = (2.0 * sh.d * (sh.K + 2) + 8 * sh.K) * sh.T / (stage_ms["combine"] / 1e3) / 1e9
    assert line["stages"]["combine"]["achieved"] == pytest.approx(comb)


def test_traffic_record_is_used_only_for_its_workload_and_source():
    fields = {}
    with open(bench.os.path.join(bench.ROOT, "profiles", "expert_ffn_traffic.txt")) as f:
        for row in f:
            if ":" in row and not row.startswith("#"):
                k, v = row.split(":", 1)
                fields[k.strip()] = v.strip()
    recorded = int(fields["dram_bytes_per_step"])
    # at least the 22.6 GB of expert weights, at most a few GB of activations more
    assert 2.25e10 < recorded < 3.0e10
    rec = bench.traffic_from_profile(synth.config("v3"))
    expected = recorded if fields["source_sha256"] == bench.kernel_source_hash() else None
    assert rec == expected
    assert bench.traffic_from_profile(synth.config("mid")) is None   # another workload


def test_decode_reports_the_weight_stream():
    _, line, _, _ = _line("decode", ffn_ms=3.1)
    assert line["roofline"]["bound"] == "hbm" and line["roofline"]["unit"] == "GB/s"
