"""Host logic of the Cache-DiT reuse decision (CPU only)."""
from __future__ import annotations

import math

import torch

from dit_block_b200.cachedit import CacheDiTPolicy, relative_change


def test_relative_change():
    sums = torch.tensor([[1.0, 4.0], [0.0, 2.0], [3.0, 0.0]], dtype=torch.float64)
    c = relative_change(sums)
    assert c[0] == 0.25 and c[1] == 0.0 and math.isinf(c[2])


def test_warmup_threshold_and_consecutive_limit():
    p = CacheDiTPolicy(threshold=0.1, warmup_steps=3, max_consecutive=2)
    # warm-up steps always recompute, whatever the change
    assert [p.decide(s, 0.0) for s in range(3)] == [False, False, False]
    # below threshold: reuse, but at most twice in a row
    assert [p.decide(s, 0.01) for s in range(3, 7)] == [True, True, False, True]
    # at or above the threshold: recompute and reset the run
    assert p.decide(7, 0.1) is False and p.consecutive == 0
    assert p.decide(8, 0.05) is True


def test_joint_decision_over_samples():
    p = CacheDiTPolicy(threshold=0.2, warmup_steps=0, max_consecutive=10)
    assert p.decide(0, [0.1, 0.15]) is True
    assert p.decide(1, [0.1, 0.25]) is False  # one sample over the threshold: all recompute
    assert p.decide(2, torch.tensor([0.01, float("inf")])) is False
