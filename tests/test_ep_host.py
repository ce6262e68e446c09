"""Host-side checks of the expert-parallel layer that run before any device
work: batch and expert counts that do not split over the ranks, and option
combinations that have no kernel path, are refused with ValueError."""
import pytest
import torch

import synth


def test_emulation_refuses_uneven_splits():
    from combine_expert_ffn_b200 import ep
    sh = synth.config("tiny")                 # T 64, E 16
    inp = {"x": torch.empty(sh.T, sh.d, dtype=torch.bfloat16)}
    with pytest.raises(ValueError):
        ep.EmulatedEP(sh, inp, 3)              # 64 % 3 != 0
    with pytest.raises(ValueError):
        ep.EmulatedEP(sh.replace(T=96), inp, 3)  # E 16 % 3 != 0


def test_dedup_combine_needs_the_dedup_dispatch():
    import combine_expert_ffn_b200 as moe
    from combine_expert_ffn_b200 import ep
    cfg = moe.MoeConfig.of(synth.config("tiny"))
    with pytest.raises(ValueError):
        ep._RankState(cfg, 2, "cpu", dedup=False, dedup_combine=True)
