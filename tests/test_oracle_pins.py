"""Pins for the fp64 CPU oracle (CPU only, no GPU).

The oracle is trusted only because it agrees with things other than itself:
  * hand-worked fixtures under tests/golden/ (budget counts, selection cases);
  * brute-force dense attention in torch fp64 with explicit boolean masks,
    and torch's scaled_dot_product_attention given the same masks;
  * closed forms (uniform weights, W = 1, constant V, zero queries, a
    three-key example with weights 1 : e : e^2);
  * invariants of the method (ratio 0, ratio 1 with W >= L, positions inside
    the window, head permutations inside a GQA group);
  * a brute-force Python sort for the selection rule.

Sources of the method (page titles and sections):
  "LoGo: Token-Level Dynamic Local-Global Attention", Abstract;
  "Learning When to Attend", "The Architecture of Conditional Attention";
  "Local-global attention", Variants (Gemma 2: causal; the windowed kind
  ignores keys further back than the window) and Implementation sketch notes
  (packed examples).
"""
import math
import os
import random

import pytest
import torch

import oracle
from token_level_dynamic_seq_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# independent brute-force references (written from the definitions)
# --------------------------------------------------------------------------

def brute_select(g, ratio):
    """Sort by (NaN last, logit descending, position ascending); keep k."""
    vals = [float(x) for x in g]
    k = oracle.num_selected(ratio, len(vals))
    order = sorted(range(len(vals)), key=lambda i: (math.isnan(vals[i]),
                                                     0.0 if math.isnan(vals[i]) else -vals[i], i))
    return sorted(order[:k])


def dense_reference(q, k, v, g, W, sel_sets, scale=None, cu_seqlens=None):
    """Dense masked attention in torch fp64: returns (local, global, out).

    local uses mask M_L[i, j] = (j <= i) and (i - j < W); global uses
    M_G[i, j] = (j <= i); both inside one sequence.  out = local +
    sigmoid(g) * global on selected rows.
    """
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    qd, kd, vd, gd = q.double(), k.double(), v.double(), g.double()
    loc = torch.zeros(B, Hq, L, d, dtype=torch.float64)
    glo = torch.zeros_like(loc)
    out = torch.zeros_like(loc)
    if cu_seqlens is None:
        spans = [(b, 0, L) for b in range(B)]
    else:
        spans = [(0, int(cu_seqlens[s]), int(cu_seqlens[s + 1])) for s in range(len(cu_seqlens) - 1)]
    for si, (b, lo, hi) in enumerate(spans):
        n = hi - lo
        if n == 0:
            continue
        i = torch.arange(n).view(-1, 1)
        j = torch.arange(n).view(1, -1)
        m_g = j <= i
        m_l = m_g & ((i - j) < W)
        sel = torch.zeros(n, dtype=torch.bool)
        sel[list(sel_sets[si])] = True
        for h in range(Hq):
            hk = h // G
            s = scale * qd[b, h, lo:hi] @ kd[b, hk, lo:hi].T
            pl = torch.softmax(s.masked_fill(~m_l, -math.inf), dim=-1)
            pg = torch.softmax(s.masked_fill(~m_g, -math.inf), dim=-1)
            lo_o = pl @ vd[b, hk, lo:hi]
            gl_o = pg @ vd[b, hk, lo:hi]
            loc[b, h, lo:hi] = lo_o
            glo[b, h, lo:hi] = torch.where(sel.view(-1, 1), gl_o, torch.zeros_like(gl_o))
            out[b, h, lo:hi] = lo_o + torch.where(
                sel.view(-1, 1), torch.sigmoid(gd[b, lo:hi]).view(-1, 1) * gl_o, torch.zeros_like(gl_o))
    return loc, glo, out


def oracle_sel_sets(res, nseq):
    cu = res["cu_sel"].tolist()
    idx = res["sel_idx"].tolist()
    return [idx[cu[s]:cu[s + 1]] for s in range(nseq)]


def rand_bf16(gen, *shape, scale=1.0):
    return (torch.randn(*shape, generator=gen) * scale).to(torch.bfloat16)


# --------------------------------------------------------------------------
# budget count and selection
# --------------------------------------------------------------------------

def read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip() if not name.startswith("select") else line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append(line)
    return rows


def test_num_selected_golden():
    for line in read_table("num_selected.txt"):
        r, n, k = line.split()[:3]
        assert oracle.num_selected(float(r), int(n)) == int(k), line


def _parse_float(tok):
    return float(tok.strip())


def test_select_golden():
    for line in read_table("select_cases.txt"):
        ratio, logits, expect = [x.strip() for x in line.split("|")]
        g = torch.tensor([_parse_float(t) for t in logits.split(",")], dtype=torch.float32)
        want = [int(t) for t in expect.split(",")] if expect else []
        got = oracle.select(g, float(ratio)).tolist()
        assert got == want, line


@pytest.mark.parametrize("seed", range(12))
def test_select_bruteforce_ties_nan_inf(seed):
    rng = random.Random(seed)
    n = rng.choice([1, 2, 7, 64, 257, 1000])
    # few distinct values so ties are everywhere; sprinkle specials
    pool = [0.0, -0.0, 1.5, -1.5, 2.0, float("inf"), float("-inf"), float("nan"), 1e-45, -1e-45]
    vals = [rng.choice(pool) if rng.random() < 0.5 else round(rng.gauss(0, 1), 1) for _ in range(n)]
    g = torch.tensor(vals, dtype=torch.float32)
    for ratio in (0.0, 0.05, 0.2, 0.25, 0.5, 0.99, 1.0):
        assert oracle.select(g, ratio).tolist() == brute_select(g.tolist(), ratio)


def test_select_matches_stable_sort():
    gen = torch.Generator().manual_seed(3)
    g = torch.randn(5000, generator=gen).to(torch.float32)
    g[::7] = g[3]  # many exact ties
    k = oracle.num_selected(0.2, g.numel())
    order = torch.sort(-g.double(), stable=True).indices[:k]
    assert oracle.select(g, 0.2).tolist() == sorted(order.tolist())


# --------------------------------------------------------------------------
# attention: brute-force dense masks and a library routine
# --------------------------------------------------------------------------

SHAPES = [
    # B, Hq, Hkv, L, d, W, ratio
    (1, 2, 2, 40, 16, 5, 0.25),
    (2, 4, 2, 33, 8, 7, 0.2),
    (1, 8, 2, 50, 32, 64, 0.5),    # W >= L
    (1, 3, 1, 17, 4, 1, 0.3),      # W = 1
    (2, 2, 2, 1, 8, 4, 1.0),       # L = 1
]


@pytest.mark.parametrize("shape", SHAPES)
def test_oracle_vs_dense_masks(shape):
    B, Hq, Hkv, L, d, W, ratio = shape
    gen = torch.Generator().manual_seed(int(sum(shape[:6])))
    q = rand_bf16(gen, B, Hq, L, d)
    k = rand_bf16(gen, B, Hkv, L, d)
    v = rand_bf16(gen, B, Hkv, L, d)
    g = torch.randn(B, L, generator=gen)
    res = oracle.forward(q, k, v, g, W, ratio, want_branches=True)
    sets = [brute_select(g[b].tolist(), ratio) for b in range(B)]
    assert oracle_sel_sets(res, B) == sets
    loc, glo, out = dense_reference(q, k, v, g, W, sets)
    torch.testing.assert_close(res["local"], loc, rtol=1e-12, atol=1e-12)
    torch.testing.assert_close(res["global"], glo, rtol=1e-12, atol=1e-12)
    torch.testing.assert_close(res["out"], out, rtol=1e-12, atol=1e-12)


def test_oracle_vs_dense_masks_varlen():
    gen = torch.Generator().manual_seed(11)
    lens = [5, 1, 0, 23, 12]
    T = sum(lens)
    cu = torch.tensor([0] + list(torch.cumsum(torch.tensor(lens), 0)), dtype=torch.int32)
    q = rand_bf16(gen, 1, 4, T, 16)
    k = rand_bf16(gen, 1, 2, T, 16)
    v = rand_bf16(gen, 1, 2, T, 16)
    g = torch.randn(1, T, generator=gen)
    W, ratio = 4, 0.25
    res = oracle.forward(q, k, v, g, W, ratio, cu_seqlens=cu, want_branches=True)
    sets = [brute_select(g[0, int(cu[s]):int(cu[s + 1])].tolist(), ratio) for s in range(len(lens))]
    assert oracle_sel_sets(res, len(lens)) == sets
    loc, glo, out = dense_reference(q, k, v, g, W, sets, cu_seqlens=cu)
    torch.testing.assert_close(res["out"], out, rtol=1e-12, atol=1e-12)
    torch.testing.assert_close(res["local"], loc, rtol=1e-12, atol=1e-12)


def test_oracle_vs_sdpa():
    gen = torch.Generator().manual_seed(5)
    B, Hq, Hkv, L, d, W = 1, 4, 4, 48, 32, 9
    q = rand_bf16(gen, B, Hq, L, d)
    k = rand_bf16(gen, B, Hkv, L, d)
    v = rand_bf16(gen, B, Hkv, L, d)
    g = torch.randn(B, L, generator=gen)
    res = oracle.forward(q, k, v, g, W, 1.0, want_branches=True)
    i = torch.arange(L).view(-1, 1)
    j = torch.arange(L).view(1, -1)
    m_l = (j <= i) & (i - j < W)
    m_g = j <= i
    sd = torch.nn.functional.scaled_dot_product_attention
    loc = sd(q.double(), k.double(), v.double(), attn_mask=m_l)
    glo = sd(q.double(), k.double(), v.double(), attn_mask=m_g)
    torch.testing.assert_close(res["local"], loc, rtol=1e-12, atol=1e-12)
    torch.testing.assert_close(res["global"], glo, rtol=1e-12, atol=1e-12)


def test_oracle_custom_scale():
    gen = torch.Generator().manual_seed(6)
    q = rand_bf16(gen, 1, 2, 20, 8)
    k = rand_bf16(gen, 1, 2, 20, 8)
    v = rand_bf16(gen, 1, 2, 20, 8)
    g = torch.randn(1, 20, generator=gen)
    res = oracle.forward(q, k, v, g, 6, 0.5, scale=0.37, want_branches=True)
    sets = [brute_select(g[0].tolist(), 0.5)]
    loc, glo, out = dense_reference(q, k, v, g, 6, sets, scale=0.37)
    torch.testing.assert_close(res["out"], out, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------

def test_closed_form_uniform_weights():
    # q = 0 makes every score 0, so each branch is a plain mean of V rows.
    # V rows (d = 2): [1, 0], [2, -2], [4, 8]; W = 2; gates all 0, k = 1.
    # local: row0 = [1,0]; row1 = mean(v0,v1) = [1.5,-1]; row2 = mean(v1,v2) = [3,3].
    # selection: all logits tie, so position 0; global(row0) = v0; sigmoid(0) = 1/2.
    # out: row0 = [1,0] + [0.5,0] = [1.5,0]; rows 1, 2 = local.
    q = torch.zeros(1, 1, 3, 2, dtype=torch.bfloat16)
    k = torch.tensor([[[[1.0, 2.0], [3.0, -1.0], [0.5, 0.25]]]], dtype=torch.bfloat16)
    v = torch.tensor([[[[1.0, 0.0], [2.0, -2.0], [4.0, 8.0]]]], dtype=torch.bfloat16)
    g = torch.zeros(1, 3)
    res = oracle.forward(q, k, v, g, 2, 1.0 / 3.0, want_branches=True)
    assert res["sel_idx"].tolist() == [0]
    want = torch.tensor([[1.5, 0.0], [1.5, -1.0], [3.0, 3.0]], dtype=torch.float64)
    torch.testing.assert_close(res["out"][0, 0], want, rtol=0, atol=1e-15)


def test_closed_form_weights_one_e_e2():
    # scale 1, q_2 = [1, 0], keys [0,0], [1,0], [2,0]: scores 0, 1, 2, so the
    # global weights of row 2 are 1 : e : e^2.  With v0 = [1,0], v1 = [0,1],
    # v2 = [0,0]: global_2 = [1, e] / (1 + e + e^2).  W = 2 keeps keys 1, 2:
    # local_2 = [0, e] / (e + e^2) = [0, 1/(1+e)].
    q = torch.tensor([[[[0.0, 0.0], [0.0, 0.0], [1.0, 0.0]]]], dtype=torch.bfloat16)
    k = torch.tensor([[[[0.0, 0.0], [1.0, 0.0], [2.0, 0.0]]]], dtype=torch.bfloat16)
    v = torch.tensor([[[[1.0, 0.0], [0.0, 1.0], [0.0, 0.0]]]], dtype=torch.bfloat16)
    g = torch.tensor([[0.0, 0.0, 5.0]])
    res = oracle.forward(q, k, v, g, 2, 1.0 / 3.0, scale=1.0, want_branches=True)
    e = math.e
    den = 1 + e + e * e
    assert res["sel_idx"].tolist() == [2]
    glo = torch.tensor([1 / den, e / den], dtype=torch.float64)
    loc = torch.tensor([0.0, 1 / (1 + e)], dtype=torch.float64)
    torch.testing.assert_close(res["global"][0, 0, 2], glo, rtol=1e-14, atol=1e-15)
    torch.testing.assert_close(res["local"][0, 0, 2], loc, rtol=1e-14, atol=1e-15)
    sig = 1 / (1 + math.exp(-5.0))
    torch.testing.assert_close(res["out"][0, 0, 2], loc + sig * glo, rtol=1e-14, atol=1e-15)


def _small(seed, B=1, Hq=4, Hkv=2, L=37, d=16):
    gen = torch.Generator().manual_seed(seed)
    return (rand_bf16(gen, B, Hq, L, d), rand_bf16(gen, B, Hkv, L, d), rand_bf16(gen, B, Hkv, L, d),
            torch.randn(B, L, generator=gen))


def test_window_one_is_identity_on_v():
    q, k, v, g = _small(1)
    res = oracle.forward(q, k, v, g, 1, 0.0, want_branches=True)
    G = q.shape[1] // k.shape[1]
    want = v.double().repeat_interleave(G, dim=1)
    assert torch.equal(res["local"], want)


def test_constant_v():
    q, k, v, g = _small(2)
    c = torch.tensor([0.75, -2.0]).view(1, 2, 1, 1)
    v = (torch.ones_like(v, dtype=torch.float32) * c).to(torch.bfloat16)
    res = oracle.forward(q, k, v, g, 5, 0.3)
    G = 2
    sel = set(res["sel_idx"].tolist())
    for h in range(4):
        cv = float(c.flatten()[h // G])
        for i in range(q.shape[2]):
            f = 1.0 + (1.0 / (1.0 + math.exp(-float(g[0, i]))) if i in sel else 0.0)
            assert torch.allclose(res["out"][0, h, i], torch.full((16,), cv * f, dtype=torch.float64),
                                  rtol=1e-13, atol=1e-13)


def test_zero_q_gives_window_mean():
    q, k, v, g = _small(3)
    q = torch.zeros_like(q)
    W = 6
    res = oracle.forward(q, k, v, g, W, 0.0, want_branches=True)
    vd = v.double()
    for h in range(4):
        for i in range(q.shape[2]):
            lo = max(0, i - W + 1)
            want = vd[0, h // 2, lo:i + 1].mean(0)
            torch.testing.assert_close(res["local"][0, h, i], want, rtol=1e-13, atol=1e-14)


# --------------------------------------------------------------------------
# invariants of the method
# --------------------------------------------------------------------------

def test_ratio_zero_is_pure_local():
    q, k, v, g = _small(4)
    res = oracle.forward(q, k, v, g, 7, 0.0, want_branches=True)
    assert res["sel_idx"].numel() == 0
    assert torch.equal(res["out"], res["local"])


def test_ratio_one_full_window_is_gated_causal():
    q, k, v, g = _small(5)
    L = q.shape[2]
    res = oracle.forward(q, k, v, g, L, 1.0, want_branches=True)
    causal = torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double().repeat_interleave(2, 1), v.double().repeat_interleave(2, 1),
        is_causal=True)
    want = causal * (1.0 + torch.sigmoid(g.double())).view(1, 1, L, 1)
    torch.testing.assert_close(res["out"], want, rtol=1e-12, atol=1e-12)


def test_selected_inside_window_doubles_local():
    q, k, v, g = _small(6, L=64)
    W = 20
    res = oracle.forward(q, k, v, g, W, 0.5, want_branches=True)
    for i in res["sel_idx"].tolist():
        if i < W:
            f = 1.0 + 1.0 / (1.0 + math.exp(-float(g[0, i])))
            torch.testing.assert_close(res["out"][0, :, i], f * res["local"][0, :, i],
                                       rtol=1e-12, atol=1e-13)


def test_head_permutation_within_group_commutes():
    q, k, v, g = _small(7, Hq=6, Hkv=2)
    res = oracle.forward(q, k, v, g, 9, 0.25)
    perm = [2, 0, 1, 5, 3, 4]  # permutes heads inside each group of 3
    res_p = oracle.forward(q[:, perm].contiguous(), k, v, g, 9, 0.25)
    torch.testing.assert_close(res_p["out"], res["out"][:, perm], rtol=0, atol=0)


def test_rows_matches_forward():
    w = workloads.load("tiny")
    res = oracle.forward(w.q, w.k, w.v, w.g, w.W, w.ratio, want_branches=True)
    sel = set(res["sel_idx"].tolist())
    rng = random.Random(0)
    picks = [(0, rng.randrange(w.Hq), rng.randrange(w.L)) for _ in range(40)]
    loc, glo, out = oracle.rows(w.q, w.k, w.v, w.g, w.W, [p[0] for p in picks], [p[1] for p in picks],
                                [p[2] for p in picks], [int(p[2] in sel) for p in picks])
    for t, (_, h, i) in enumerate(picks):
        assert torch.equal(out[t], res["out"][0, h, i])
        assert torch.equal(loc[t], res["local"][0, h, i])
