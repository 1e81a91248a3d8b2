"""Pins for the oracle's decode step (CPU only).

The new token of each sequence sits at the end of its key/value cache; its
local branch reads the last W positions, and it reads the whole cache only if
its gate logit passes the threshold.  Pins: a dense torch fp64 reference with
explicit masks, agreement with the prefill oracle's row for the same token
(threshold set to the controller target, so selections agree), and closed
forms (empty cache, W = 1).
"""
import math

import pytest
import torch

import oracle


def dense_decode(q, k, v, cache_len, g, tau, W):
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(d)
    out = torch.zeros(B, Hq, d, dtype=torch.float64)
    for b in range(B):
        t = int(cache_len[b]) - 1
        if t < 0:
            continue
        sel = (not math.isnan(float(g[b]))) and (not math.isnan(tau)) and float(g[b]) > tau
        j = torch.arange(t + 1)
        m_loc = j >= t - W + 1
        for h in range(Hq):
            kk = k[b, h // G, :t + 1].double()
            vv = v[b, h // G, :t + 1].double()
            s = scale * (kk @ q[b, h].double())
            loc = torch.softmax(s.masked_fill(~m_loc, -math.inf), 0) @ vv
            o = loc
            if sel:
                o = loc + torch.sigmoid(torch.tensor(float(g[b]), dtype=torch.float64)) * (torch.softmax(s, 0) @ vv)
            out[b, h] = o
    return out


@pytest.mark.parametrize("seed", range(4))
def test_decode_vs_dense_masks(seed):
    gen = torch.Generator().manual_seed(seed)
    B, Hq, Hkv, Lmax, d, W = 5, 4, 2, 40, 16, 7
    q = torch.randn(B, Hq, d, generator=gen).bfloat16()
    k = torch.randn(B, Hkv, Lmax, d, generator=gen).bfloat16()
    v = torch.randn(B, Hkv, Lmax, d, generator=gen).bfloat16()
    cache_len = torch.tensor([40, 1, 7, 23, 8], dtype=torch.int32)
    g = torch.randn(B, generator=gen)
    tau = 0.1
    out, loc, glo, sel = oracle.decode(q, k, v, cache_len, g, tau, W)
    torch.testing.assert_close(out, dense_decode(q, k, v, cache_len, g, tau, W), rtol=1e-12, atol=1e-12)
    assert sel.tolist() == [int(float(x) > tau) for x in g]


def test_decode_matches_prefill_rows():
    gen = torch.Generator().manual_seed(9)
    Hq, Hkv, L, d, W, ratio = 4, 2, 48, 16, 9, 0.25
    q = torch.randn(1, Hq, L, d, generator=gen).bfloat16()
    k = torch.randn(1, Hkv, L, d, generator=gen).bfloat16()
    v = torch.randn(1, Hkv, L, d, generator=gen).bfloat16()
    g = torch.randn(1, L, generator=gen)
    pre = oracle.forward(q, k, v, g, W, ratio)["out"]
    tau = oracle.threshold_target(g[0], ratio)
    for t in range(L):
        out, _, _, sel = oracle.decode(q[:, :, t], k, v, torch.tensor([t + 1], dtype=torch.int32), g[:, t], tau, W)
        assert bool(sel[0]) == (t in set(oracle.select(g[0], ratio).tolist()))
        torch.testing.assert_close(out[0], pre[0, :, t], rtol=0, atol=0)


def test_decode_closed_forms():
    gen = torch.Generator().manual_seed(2)
    q = torch.randn(2, 2, 8, generator=gen).bfloat16()
    k = torch.randn(2, 1, 6, 8, generator=gen).bfloat16()
    v = torch.randn(2, 1, 6, 8, generator=gen).bfloat16()
    out, loc, glo, sel = oracle.decode(q, k, v, torch.tensor([0, 6], dtype=torch.int32),
                                       torch.tensor([5.0, -5.0]), 0.0, 1)
    assert torch.equal(out[0], torch.zeros(2, 8, dtype=torch.float64))   # empty cache
    assert torch.equal(loc[1], v[1, 0, 5].double().expand(2, 8))          # W = 1: the token's own value
    assert sel.tolist() == [1, 0]
