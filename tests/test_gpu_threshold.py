"""Threshold form of the budget rule on the GPU, against the oracle (bit-exact).

"LoGo: Token-Level Dynamic Local-Global Attention", Abstract: the share of
global tokens is held by a controller that moves a threshold on the gate.
Selections and the controller's target / updated threshold are integer or
exactly-rounded fp32 results, so they must match the oracle bit for bit.
"""
import math
import os
import random

import pytest
import torch

import oracle
import token_level_dynamic_seq_b200 as logo
from token_level_dynamic_seq_b200 import workloads

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "threshold_cases.txt")


def _shape_1d(n, cu=None, nseq=1, max_len=None):
    return logo.Shape(1, 1, 1, n, 128, None if cu is None else cu.data_ptr(), nseq,
                      n if max_len is None else max_len)


def _gpu_select(g_cpu, tau, cap=None, cu=None, seqlens=None):
    g = g_cpu.reshape(1, -1).cuda()
    n = g.shape[1]
    cu_d = None if cu is None else cu.cuda()
    nseq = 1 if cu is None else cu.numel() - 1
    ml = n if seqlens is None else max(seqlens)
    cap = ml if cap is None else cap
    sh = _shape_1d(n, cu_d, nseq, ml)
    ws = logo.workspace(sh, 0.5, g.device)
    tau_d = torch.tensor([tau], dtype=torch.float32, device="cuda")
    sel, cu_sel = logo.select_threshold(g, sh, tau_d, cap, ws)
    return sel, cu_sel, ws


def test_threshold_golden_on_gpu():
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        kind, logits, par, want = [x.strip() for x in line.split("|")]
        g = torch.tensor([float(t) for t in logits.split(",")], dtype=torch.float32)
        if kind == "select":
            sel, cu_sel, ws = _gpu_select(g, float(par))
            logo.check(ws)
            got = sel[:int(cu_sel[1])].cpu().tolist()
            assert got == oracle.threshold_select(g, float(par)).tolist(), line
        else:
            gd = g.reshape(1, -1).cuda()
            sh = _shape_1d(g.numel())
            ws = logo.workspace(sh, 0.5, gd.device)
            tau = torch.tensor([0.0], dtype=torch.float32, device="cuda")
            tgt = logo.threshold_update(gd, sh, float(par), 1.0, tau, ws)
            logo.check(ws)
            assert float(tgt.item()) == float(want) == oracle.threshold_target(g, float(par)), line
            assert float(tau.item()) == float(want), line


@pytest.mark.parametrize("seed", range(5))
def test_threshold_select_random_varlen(seed):
    rng = random.Random(seed)
    lens = [rng.choice([0, 1, 7, 1000, 4097, 30000]) for _ in range(rng.randint(1, 6))]
    cu = torch.tensor([0] + list(torch.cumsum(torch.tensor(lens), 0)), dtype=torch.int32)
    gen = torch.Generator().manual_seed(seed)
    g = (torch.randn(sum(lens), generator=gen) * 4).round() / 4
    if g.numel():
        idx = torch.randint(0, g.numel(), (max(1, g.numel() // 40),), generator=gen)
        specials = torch.tensor([0.0, -0.0, float("inf"), float("-inf"), float("nan")])
        g[idx] = specials[torch.randint(0, 5, (idx.numel(),), generator=gen)]
    for tau in (0.0, 0.75, -1.25, float("-inf"), float("nan")):
        sel, cu_sel, ws = _gpu_select(g, tau, cu=cu, seqlens=lens)
        logo.check(ws)
        cs = cu_sel.cpu().tolist()
        for s, n in enumerate(lens):
            want = oracle.threshold_select(g[int(cu[s]):int(cu[s + 1])], tau).tolist()
            assert sel[cs[s]:cs[s + 1]].cpu().tolist() == want


def test_threshold_capacity_is_reported():
    g = torch.arange(100, dtype=torch.float32)
    sel, cu_sel, ws = _gpu_select(g, 49.5, cap=10)
    with pytest.raises(logo.LogoError) as e:
        logo.check(ws)
    assert e.value.status == 6
    assert sel[:int(cu_sel[1])].cpu().tolist() == list(range(50, 60))  # lowest positions kept


@pytest.mark.parametrize("name", ["c32k", "varlen"])
def test_controller_step_matches_oracle(name):
    w = workloads.load(name)
    g = w.g.cuda()
    cu = None if w.cu_seqlens is None else w.cu_seqlens.cuda()
    sh = logo.Shape(w.B, w.Hq, w.Hkv, w.L, w.d, None if cu is None else cu.data_ptr(), len(w.seqlens),
                    max(w.seqlens))
    ws = logo.workspace(sh, w.ratio, g.device)
    flat = w.g.flatten() if w.cu_seqlens is None else w.g[0, :int(w.cu_seqlens[-1])]
    tau_host = 0.3
    tau = torch.tensor([tau_host], dtype=torch.float32, device="cuda")
    for beta in (0.25, 1.0):
        tgt = logo.threshold_update(g, sh, w.ratio, beta, tau, ws)
        logo.check(ws)
        q = oracle.threshold_target(flat, w.ratio)
        tau_host = oracle.threshold_update(tau_host, q, beta)
        assert float(tgt.item()) == q
        assert float(tau.item()) == tau_host
    # after the beta = 1 step every sequence's selection at tau reproduces the oracle's
    cap = max(w.seqlens)
    sel, cu_sel = logo.select_threshold(g, sh, tau, cap, ws)
    logo.check(ws)
    cs = cu_sel.cpu().tolist()
    total = 0
    for s, n in enumerate(w.seqlens):
        lo = 0 if w.cu_seqlens is None else int(w.cu_seqlens[s])
        row = w.g[s] if w.cu_seqlens is None else w.g[0, lo:lo + n]
        want = oracle.threshold_select(row, tau_host).tolist()
        assert sel[cs[s]:cs[s + 1]].cpu().tolist() == want
        total += len(want)
    # the target leaves at most k logits of the batch above it (exactly k without ties)
    assert total <= oracle.num_selected(w.ratio, flat.numel())
