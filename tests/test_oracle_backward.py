"""Pins for the oracle's backward pass (CPU only, no GPU).

The backward is the chain rule through the forward definition, with one
reading: the output depends on a gate logit only through the sigmoid factor
on selected rows (the selection itself is a step function and passes no
gradient).  It is trusted because it agrees with things other than itself:
  * finite differences of the oracle's forward pass (already pinned by
    tests/test_oracle_pins.py), taken with a five-point stencil on inputs and
    steps that bf16 represents exactly, so the forward sees the perturbed
    values without rounding;
  * torch autograd through torch's scaled_dot_product_attention (fp64) with
    the window and causal masks, and through the sigmoid merge;
  * invariants: the key gradients of one softmax row sum to zero, so the
    key gradient of a whole key/value head sums to zero; the value gradient
    of a head sums to the sum of the upstream gradients it received
    (1 + sigmoid(g) on selected rows); the gate gradient is zero off the
    selection.

Sources of the method (page titles and sections): "LoGo: Token-Level Dynamic
Local-Global Attention", Abstract (a learned gate, trained with the rest of
the model, no auxiliary loss); "Learning When to Attend", "The Architecture
of Conditional Attention" and "Empirical Validation and System Optimization"
(trained end to end; training throughput).
"""
import math

import pytest
import torch
import torch.nn.functional as F

import oracle
from token_level_dynamic_seq_b200 import workloads

STEP = 2.0 ** -6  # every multiple of 2^-6 in [-2, 2] is exact in bf16


def grid_bf16(gen, *shape, lim=1.0):
    """Random multiples of 2^-6 in [-lim, lim] (exact in bf16)."""
    n = int(round(lim / STEP))
    return (torch.randint(-n, n + 1, shape, generator=gen).double() * STEP).bfloat16()


def spaced_gate(gen, B, L):
    """Distinct fp32 logits at least 2^-4 apart, so a 2^-10 step never changes the selection."""
    g = torch.empty(B, L)
    for b in range(B):
        g[b] = (torch.randperm(L, generator=gen).double() * 2.0 ** -4 - L * 2.0 ** -5).float()
    return g


def make(seed, B, Hq, Hkv, L, d, cu=None):
    gen = torch.Generator().manual_seed(seed)
    q = grid_bf16(gen, B, Hq, L, d, lim=1.5)
    k = grid_bf16(gen, B, Hkv, L, d, lim=1.5)
    v = grid_bf16(gen, B, Hkv, L, d)
    g = spaced_gate(gen, B, L)
    e = grid_bf16(gen, B, Hq, L, d)
    return q, k, v, g, e


def loss(q, k, v, g, e, W, ratio, cu):
    out = oracle.forward(q, k, v, g, W, ratio, cu_seqlens=cu)["out"]
    return float((out * e.double()).sum())


def fd_grad(x, f, step):
    """Five-point central difference of f at every element of x (x is modified and restored)."""
    flat = x.view(-1)
    grad = torch.zeros(flat.numel(), dtype=torch.float64)
    for t in range(flat.numel()):
        x0 = flat[t].clone()
        vals = []
        for m in (-2, -1, 1, 2):
            flat[t] = (x0.double() + m * step).to(x.dtype)
            assert float(flat[t]) == float(x0) + m * step  # exact step
            vals.append(f())
        flat[t] = x0
        grad[t] = (vals[0] - 8 * vals[1] + 8 * vals[2] - vals[3]) / (12 * step)
    return grad.view(x.shape)


FD_CASES = [
    # seed, B, Hq, Hkv, L, d, W, ratio, seqlens (packed) or None
    (0, 1, 2, 1, 9, 4, 3, 0.34, None),     # GQA 2:1, both branches
    (1, 2, 2, 2, 7, 3, 2, 0.5, None),      # MHA, two batch rows
    (2, 1, 3, 1, 8, 2, 100, 1.0, None),    # every row global, window covers all
    (3, 1, 2, 1, 6, 4, 1, 0.0, None),      # W = 1, no global rows
    (4, 1, 2, 1, 0, 3, 2, 0.4, [5, 1, 4]), # packed sequences
]


@pytest.mark.parametrize("case", FD_CASES)
def test_backward_matches_finite_differences(case):
    seed, B, Hq, Hkv, L, d, W, ratio, lens = case
    cu = None
    if lens is not None:
        L = sum(lens)
        cu = torch.tensor([0] + list(torch.cumsum(torch.tensor(lens), 0)), dtype=torch.int32)
    q, k, v, g, e = make(seed, B, Hq, Hkv, L, d)
    f = lambda: loss(q, k, v, g, e, W, ratio, cu)
    got = oracle.backward(q, k, v, g, e, W, ratio, cu_seqlens=cu)
    for name, x, step in (("dq", q, STEP), ("dk", k, STEP), ("dv", v, STEP), ("dg", g, 2.0 ** -10)):
        want = fd_grad(x, f, step)
        err = (got[name] - want).abs().max().item()
        assert err < 1e-6, f"{name}: max error {err:.3e} against finite differences"
    assert got["dg"].abs().sum() > 0 or ratio == 0.0


def sdpa_reference(q, k, v, g, e, W, sel_flags, scale=None):
    """Autograd through torch SDPA (fp64): out = SDPA(window) + sigmoid(g) * flags * SDPA(causal)."""
    B, Hq, L, d = q.shape
    G = Hq // k.shape[1]
    qd = q.double().requires_grad_()
    kd = k.double().requires_grad_()
    vd = v.double().requires_grad_()
    gd = g.double().requires_grad_()
    i = torch.arange(L).view(L, 1)
    j = torch.arange(L).view(1, L)
    causal = j <= i
    window = causal & (i - j < W)
    ke, ve = kd.repeat_interleave(G, 1), vd.repeat_interleave(G, 1)
    loc = F.scaled_dot_product_attention(qd, ke, ve, attn_mask=window, scale=scale)
    glo = F.scaled_dot_product_attention(qd, ke, ve, attn_mask=causal, scale=scale)
    gate = torch.sigmoid(gd) * sel_flags.double()
    out = loc + gate.view(B, 1, L, 1) * glo
    (out * e.double()).sum().backward()
    return qd.grad, kd.grad, vd.grad, gd.grad


@pytest.mark.parametrize("seed,W,ratio", [(0, 16, 0.2), (1, 5, 0.5), (2, 64, 0.0), (3, 1, 1.0), (4, 33, 0.13)])
def test_backward_vs_sdpa_autograd(seed, W, ratio):
    gen = torch.Generator().manual_seed(100 + seed)
    B, Hq, Hkv, L, d = 2, 4, 2, 48, 16
    q = torch.randn(B, Hq, L, d, generator=gen).bfloat16()
    k = torch.randn(B, Hkv, L, d, generator=gen).bfloat16()
    v = torch.randn(B, Hkv, L, d, generator=gen).bfloat16()
    g = torch.randn(B, L, generator=gen)
    e = torch.randn(B, Hq, L, d, generator=gen).bfloat16()
    flags = oracle.selection_flags(g, ratio)
    dq, dk, dv, dg = sdpa_reference(q, k, v, g, e, W, flags)
    got = oracle.backward(q, k, v, g, e, W, ratio)
    for name, want in (("dq", dq), ("dk", dk), ("dv", dv), ("dg", dg)):
        err = (got[name] - want).abs().max().item()
        assert err < 1e-9, f"{name}: max error {err:.3e} against SDPA autograd"


def test_backward_invariants():
    w = workloads.make(1, 6, 2, 0, 16, 9, 0.25, seed=7, qkv_scale=1.0, seqlens=[30, 1, 0, 45, 17])
    gen = torch.Generator().manual_seed(7)
    e = torch.randn(w.q.shape, generator=gen).bfloat16()
    r = oracle.backward(w.q, w.k, w.v, w.g, e, w.W, w.ratio, cu_seqlens=w.cu_seqlens)
    flags = oracle.selection_flags(w.g, w.ratio, w.cu_seqlens)[0].bool()
    G = w.Hq // w.Hkv
    cu = w.cu_seqlens.tolist()
    sg = torch.sigmoid(w.g[0].double())
    weight = 1.0 + torch.where(flags, sg, torch.zeros_like(sg))  # upstream weight per row
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if b == a:
            continue
        for hk in range(w.Hkv):
            # softmax rows: sum_j dS_ij = 0, so the key gradient of a head sums to zero
            assert r["dk"][0, hk, a:b].sum(0).abs().max() < 1e-12
            # each softmax row's probabilities sum to one
            heads = e[0, hk * G:(hk + 1) * G, a:b].double()
            want = (heads * weight[a:b].view(1, -1, 1)).sum((0, 1))
            assert (r["dv"][0, hk, a:b].sum(0) - want).abs().max() < 1e-12
    assert (r["dg"][0][~flags] == 0).all()
    assert (r["dg"][0][flags] != 0).all()


def test_backward_rows_match_full():
    w = workloads.make(2, 4, 2, 50, 8, 11, 0.3, seed=9, qkv_scale=1.0)
    gen = torch.Generator().manual_seed(9)
    e = torch.randn(w.q.shape, generator=gen).bfloat16()
    full = oracle.backward(w.q, w.k, w.v, w.g, e, w.W, w.ratio)
    qrows = [(0, 0, 0), (1, 3, 49), (0, 2, 17), (1, 1, 30)]
    krows = [(0, 0, 0), (1, 1, 49), (0, 1, 12), (1, 0, 40)]
    rr = oracle.backward_rows(w.q, w.k, w.v, w.g, e, w.W, w.ratio, qrows=qrows, krows=krows)
    for t, (s, h, i) in enumerate(qrows):
        assert torch.allclose(rr["dq"][t], full["dq"][s, h, i], atol=1e-12, rtol=0)
        assert abs(rr["dg"][t] - full["dg"][s, i]) < 1e-12
    for t, (s, hk, j) in enumerate(krows):
        assert torch.allclose(rr["dk"][t], full["dk"][s, hk, j], atol=1e-12, rtol=0)
        assert torch.allclose(rr["dv"][t], full["dv"][s, hk, j], atol=1e-12, rtol=0)
