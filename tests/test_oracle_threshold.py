"""Pins for the threshold form of the budget rule in the oracle (CPU only).

"LoGo: Token-Level Dynamic Local-Global Attention", Abstract: the share of
global tokens is held by a controller that moves a threshold on the gate.
Pins: hand-worked cases (tests/golden/threshold_cases.txt), a brute-force
Python reference, the exact fp32 arithmetic of the update reproduced with
numpy float32, and the defining property of the target (exactly k logits
above it when the logits are distinct).
"""
import math
import os
import random

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "threshold_cases.txt")


def _vals(txt):
    return [float(t) for t in txt.split(",")] if txt.strip() else []


def brute_threshold_select(vals, tau):
    f = np.float32
    return [i for i, x in enumerate(vals) if not math.isnan(x) and not math.isnan(tau) and f(x) > f(tau)]


def brute_target(vals, ratio):
    n = len(vals)
    k = oracle.num_selected(ratio, n)
    if k >= n:
        return -math.inf
    order = sorted(range(n), key=lambda i: (math.isnan(vals[i]), 0.0 if math.isnan(vals[i]) else -vals[i], i))
    q = vals[order[k]]
    return -math.inf if math.isnan(q) else q


def test_threshold_golden():
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        kind, logits, par, want = [x.strip() for x in line.split("|")]
        g = torch.tensor(_vals(logits), dtype=torch.float32)
        if kind == "select":
            assert oracle.threshold_select(g, float(par)).tolist() == [int(t) for t in _vals(want)], line
        else:
            assert oracle.threshold_target(g, float(par)) == float(want), line


@pytest.mark.parametrize("seed", range(8))
def test_threshold_select_and_target_bruteforce(seed):
    rng = random.Random(seed)
    n = rng.choice([1, 3, 16, 100, 513])
    pool = [0.0, -0.0, 1.5, -1.5, float("inf"), float("-inf"), float("nan"), 1e-45, -1e-45]
    vals = [rng.choice(pool) if rng.random() < 0.4 else round(rng.gauss(0, 1), 2) for _ in range(n)]
    vals = [float(np.float32(v)) for v in vals]
    g = torch.tensor(vals, dtype=torch.float32)
    for tau in (0.0, -0.0, 1.5, -math.inf, math.inf, math.nan, 0.37, vals[0]):
        assert oracle.threshold_select(g, tau).tolist() == brute_threshold_select(vals, tau)
    for ratio in (0.0, 0.1, 0.25, 0.5, 0.99, 1.0):
        assert oracle.threshold_target(g, ratio) == brute_target(vals, ratio)


def test_target_leaves_exactly_k_above_distinct_logits():
    gen = torch.Generator().manual_seed(4)
    g = torch.randn(10000, generator=gen)
    assert torch.unique(g).numel() == g.numel()
    for ratio in (0.05, 0.2, 0.5):
        q = oracle.threshold_target(g, ratio)
        assert int((g > q).sum()) == oracle.num_selected(ratio, g.numel())


def test_threshold_update_fp32_arithmetic():
    rng = random.Random(7)
    f = np.float32
    for _ in range(500):
        tau = f(rng.gauss(0, 3))
        q = f(rng.gauss(0, 3))
        beta = f(rng.random())
        want = f(tau + f(beta * f(q - tau)))
        assert oracle.threshold_update(float(tau), float(q), float(beta)) == float(want)
    # closed forms: beta 1 jumps to the target, beta 0 keeps tau; non-finite values jump
    assert oracle.threshold_update(0.5, 2.25, 1.0) == 2.25
    assert oracle.threshold_update(0.5, 2.25, 0.0) == 0.5
    assert oracle.threshold_update(-math.inf, 2.0, 0.1) == 2.0
    assert oracle.threshold_update(1.0, -math.inf, 0.1) == -math.inf
