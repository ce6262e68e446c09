"""The seeded generator: slices regenerate alone, distributions have the stated moments."""
import math

import numpy as np
import torch

import synth


def test_slices_regenerate_alone():
    full = synth.normal(3, 4, (6, 1000), 0.5, torch.bfloat16)
    part = synth.normal_slice(3, 4, 2 * 1000 + 17, 500, 0.5, torch.bfloat16)
    assert torch.equal(full.view(-1)[2017:2517].view(torch.int16), part.view(torch.int16))


def test_expert_slice_matches_full_tensor():
    sh = synth.config("tiny")
    inp = synth.make_inputs(sh)
    for name in ("w_gate", "w_up", "w_down"):
        assert torch.equal(inp[name][5], synth.expert_slice(sh, name, 5))


def test_normal_moments():
    z = synth.normal(0, 1, (1 << 20,), 2.0, torch.float32).double()
    assert abs(z.mean().item()) < 0.01
    assert abs(z.std().item() - 2.0) < 0.01
    assert z.abs().max().item() <= 2.0 * 2 * math.sqrt(3) + 1e-6   # Irwin-Hall(4) support


def test_distinct_tensor_ids_and_seeds_differ():
    a = synth.normal(0, 1, (4096,), 1.0, torch.float32)
    b = synth.normal(0, 2, (4096,), 1.0, torch.float32)
    c = synth.normal(1, 1, (4096,), 1.0, torch.float32)
    assert abs(torch.corrcoef(torch.stack([a, b]))[0, 1]) < 0.05
    assert abs(torch.corrcoef(torch.stack([a, c]))[0, 1]) < 0.05


def test_uniform_open_interval():
    u = synth.uniform01(0, 9, (1 << 18,))
    assert (u > 0).all() and (u < 1).all()
    assert abs(u.double().mean().item() - 0.5) < 0.005


def test_zipf_offsets_are_log_probabilities():
    off = synth.zipf_logit_offset(256, 1.2, 0).double()
    assert abs(off.exp().sum().item() - 1.0) < 1e-5
    p = off.exp().sort(descending=True).values
    r = torch.arange(1, 257, dtype=torch.float64)
    np.testing.assert_allclose((p / p[0]).numpy(), r.pow(-1.2).numpy(), rtol=1e-5)


def test_random_routing_is_valid_and_skewed():
    r = synth.random_routing(0, 4096, 64, 6, 1.2)
    assert r.shape == (4096, 6)
    assert all(len(set(row)) == 6 for row in r.tolist())
    counts = torch.bincount(r.view(-1), minlength=64)
    assert counts[0] > 4 * counts[32]
    u = torch.bincount(synth.random_routing(0, 4096, 64, 6, 0.0).view(-1), minlength=64).double()
    assert u.std() / u.mean() < 0.1


def test_workload_shapes():
    inp = synth.make_inputs(synth.config("tiny"))
    assert inp["x"].dtype == torch.bfloat16 and inp["x"].shape == (64, 128)
    assert inp["router_w"].dtype == torch.float32 and inp["bias"].shape == (16,)
    assert inp["ws_down"].shape == (1, 128, 64)
