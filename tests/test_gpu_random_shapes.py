"""Forward and backward on seeded random shapes, every element against the oracle.

Each case draws its own shape from a seeded generator: batch or packed
sequences (including empty and one-token ones), the query and key/value head
counts (GQA groups of 1 to 5, odd and even), length (not a multiple of the
128-row tile), head dimension 64 or 128, window (1, a few keys, or past the
length) and ratio (0 to 1).  Selection must match bit for bit; outputs and
gradients within the same tolerances as the fixed cases.
"""
import random

import pytest
import torch

import oracle
import token_level_dynamic_seq_b200 as logo
from token_level_dynamic_seq_b200 import workloads

from tests.test_gpu_parity import MAX_ABS, close, oracle_sel_lists, sel_lists, to_dev

pytestmark = pytest.mark.gpu


def draw_case(seed):
    rng = random.Random(1000 + seed)
    Hkv = rng.choice([1, 2, 3])
    G = rng.choice([1, 2, 3, 4, 5])
    d = rng.choice([64, 128])
    W = rng.choice([1, 2, 17, 128, 129, 300, 5000])
    ratio = rng.choice([0.0, 0.05, 0.25, 0.5, 0.999, 1.0])
    if rng.random() < 0.4:
        seqlens = [rng.choice([0, 1, 2, 127, 128, 129, rng.randrange(3, 700)]) for _ in range(rng.randrange(1, 5))]
        if sum(seqlens) == 0:
            seqlens[0] = 5
        B, L = 1, 0
    else:
        seqlens = None
        B, L = rng.choice([1, 2]), rng.randrange(1, 800)
    return B, Hkv * G, Hkv, L, d, W, ratio, seqlens


CASES = list(range(24))


@pytest.mark.parametrize("seed", CASES)
def test_forward_random_shape(seed):
    B, Hq, Hkv, L, d, W, ratio, lens = draw_case(seed)
    w = workloads.make(B, Hq, Hkv, L, d, W, ratio, seed=seed, qkv_scale=1.0, seqlens=lens, name=f"random{seed}")
    q, k, v, g, cu = to_dev(w)
    ml = max(w.seqlens)
    out, sel, cu_sel = logo.forward(q, k, v, g, w.W, w.ratio, cu_seqlens=cu, max_seqlen=ml if cu is not None else None)
    torch.cuda.synchronize()
    ref = oracle.forward(w.q, w.k, w.v, w.g, w.W, w.ratio, cu_seqlens=w.cu_seqlens)
    assert sel_lists(sel, cu_sel) == oracle_sel_lists(w)
    T = w.L if w.cu_seqlens is None else int(w.cu_seqlens[-1])
    # Unscaled N(0,1) inputs with a short window give outputs up to |o| ~ 8; the merged row is
    # rounded to bf16 twice, up to one bf16 spacing at its magnitude: the max-abs bound scales
    # with the output as in the large-output tests, 2e-2 * max(1, max|ref| / 2); rel-L2 5e-3.
    r = ref["out"][:, :, :T]
    close(out[:, :, :T], r, f"random {seed} {(B, Hq, Hkv, L, d, W, ratio, lens)}",
          max_abs=MAX_ABS * max(1.0, r.abs().max().item() / 2.0))


# seeds 120 and 184 draw W = 1 with ratio 0: every row attends to itself alone, so dQ is exactly
# zero (the one softmax weight is 1 and dP equals D); seed 360 selects one row of a 5-token
# sequence whose gate gradient sums terms that largely cancel
@pytest.mark.parametrize("seed", CASES[:12] + [120, 184, 360])
def test_backward_random_shape(seed):
    from tests.test_gpu_backward import close as close_grad, gpu_run

    B, Hq, Hkv, L, d, W, ratio, lens = draw_case(seed)
    w = workloads.make(B, Hq, Hkv, L, d, W, ratio, seed=seed, qkv_scale=1.0, seqlens=lens, name=f"random{seed}")
    e = torch.randn(w.q.shape, generator=torch.Generator().manual_seed(seed)).bfloat16()
    dq, dk, dv, dg = gpu_run(w, e)
    ref = oracle.backward(w.q, w.k, w.v, w.g, e, w.W, w.ratio, cu_seqlens=w.cu_seqlens)
    T = w.L if w.cu_seqlens is None else int(w.cu_seqlens[-1])
    what = f"random {seed} {(B, Hq, Hkv, L, d, W, ratio, lens)}"
    close_grad(dq[:, :, :T], ref["dq"][:, :, :T], what + " dq")
    close_grad(dk[:, :, :T], ref["dk"][:, :, :T], what + " dk")
    close_grad(dv[:, :, :T], ref["dv"][:, :, :T], what + " dv")
    if (ref["dg"] != 0).any():
        check_dgate(w, e, dg[:, :T], ref["dg"][:, :T], T, what + " dgate")


def check_dgate(w, e, dg, ref_dg, T, what):
    """The gate gradient of a selected row is sigma'(g) * sum over heads and columns of
    dout * global (the global branch before the gate).  The kernels form it from the bf16 global
    branch, so its error is bounded by the rounding of the terms, not by the size of the sum:
    where the terms cancel the relative error of the sum grows without bound.  The check is the
    dot product's forward-error bound with 5e-3 (about 2.5 bf16 roundings) per term:
    |dg - ref| <= 5e-3 * sigma'(g) * sum |dout * global|, row by row."""
    fwd = oracle.forward(w.q, w.k, w.v, w.g, w.W, w.ratio, cu_seqlens=w.cu_seqlens, want_branches=True)
    glob = fwd["global"][:, :, :T]
    terms = (e[:, :, :T].double() * glob).abs().sum(dim=(1, 3))  # [B, T]
    sg = torch.sigmoid(w.g[:, :T].double())
    bound = 5e-3 * sg * (1.0 - sg) * terms
    err = (dg.double().cpu() - ref_dg.double()).abs()
    worst = (err - bound).max().item()
    print(f"{what}: max-abs {err.max().item():.3e}, worst margin {worst:.3e}")
    assert (err <= bound + 1e-7).all(), f"{what}: an error above the per-row bound (margin {worst:.3e})"


MEDIUM = [
    # name, B, Hq, Hkv, L, d, W, ratio, seqlens: group sizes the named workloads do not use,
    # at sizes that span many tiles (odd groups pair consecutive row tiles in one CTA)
    ("odd group 3 varlen", 1, 6, 2, 0, 128, 700, 0.2, [3000, 1, 5000, 129]),
    ("group 8", 1, 16, 2, 2500, 128, 1024, 0.25, None),
    ("odd group 5 d64", 2, 5, 1, 1800, 64, 300, 0.3, None),
]


@pytest.mark.parametrize("case", MEDIUM, ids=[c[0] for c in MEDIUM])
def test_forward_medium_edge_groups(case):
    name, B, Hq, Hkv, L, d, W, ratio, lens = case
    w = workloads.make(B, Hq, Hkv, L, d, W, ratio, seed=7, qkv_scale=1.0, seqlens=lens, name=name)
    q, k, v, g, cu = to_dev(w)
    ml = max(w.seqlens)
    out, sel, cu_sel = logo.forward(q, k, v, g, w.W, w.ratio, cu_seqlens=cu, max_seqlen=ml if cu is not None else None)
    torch.cuda.synchronize()
    ref = oracle.forward(w.q, w.k, w.v, w.g, w.W, w.ratio, cu_seqlens=w.cu_seqlens)
    assert sel_lists(sel, cu_sel) == oracle_sel_lists(w)
    T = w.L if w.cu_seqlens is None else int(w.cu_seqlens[-1])
    r = ref["out"][:, :, :T]
    close(out[:, :, :T], r, name, max_abs=MAX_ABS * max(1.0, r.abs().max().item() / 2.0))


def draw_medium(seed):
    """A seeded shape of a few thousand tokens: group sizes 1 to 8, d 64 or 128, windows from 64
    to 8192 and ratios from 0.02 to 1, fixed-length batches or 2 to 5 packed sequences."""
    rng = random.Random(5000 + seed)
    Hkv = rng.choice([1, 2])
    G = rng.choice([1, 2, 3, 4, 6, 8])
    d = rng.choice([64, 128])
    W = rng.choice([64, 500, 1024, 2047, 4096, 8192])
    ratio = rng.choice([0.02, 0.1, 0.2, 0.33, 0.6, 1.0])
    if rng.random() < 0.4:
        seqlens = [rng.randrange(1, 6000) for _ in range(rng.randrange(2, 6))]
        return 1, Hkv * G, Hkv, 0, d, W, ratio, seqlens
    return rng.choice([1, 2]), Hkv * G, Hkv, rng.randrange(1000, 9000), d, W, ratio, None


@pytest.mark.parametrize("seed", range(8))
def test_forward_medium_random_shape(seed):
    """Every element at sizes that span many CTAs of both launches and ragged tails."""
    B, Hq, Hkv, L, d, W, ratio, lens = draw_medium(seed)
    w = workloads.make(B, Hq, Hkv, L, d, W, ratio, seed=seed, seqlens=lens, name=f"medium{seed}")
    q, k, v, g, cu = to_dev(w)
    ml = max(w.seqlens)
    out, sel, cu_sel = logo.forward(q, k, v, g, w.W, w.ratio, cu_seqlens=cu, max_seqlen=ml if cu is not None else None)
    torch.cuda.synchronize()
    ref = oracle.forward(w.q, w.k, w.v, w.g, w.W, w.ratio, cu_seqlens=w.cu_seqlens)
    assert sel_lists(sel, cu_sel) == oracle_sel_lists(w)
    T = w.L if w.cu_seqlens is None else int(w.cu_seqlens[-1])
    r = ref["out"][:, :, :T]
    close(out[:, :, :T], r, f"medium {seed} {(B, Hq, Hkv, L, d, W, ratio, lens)}",
          max_abs=MAX_ABS * max(1.0, r.abs().max().item() / 2.0))


def draw_medium_backward(seed):
    """A seeded shape of 500 to 3000 tokens for the backward: group sizes 1 to 8, d 64 or 128,
    windows 64 to 4096, ratios 0.05 to 1, fixed-length batches or 2 to 4 packed sequences."""
    rng = random.Random(7000 + seed)
    Hkv = rng.choice([1, 2])
    G = rng.choice([1, 2, 3, 4, 8])
    d = rng.choice([64, 128])
    W = rng.choice([64, 300, 1024, 4096])
    ratio = rng.choice([0.05, 0.2, 0.5, 1.0])
    if rng.random() < 0.4:
        return 1, Hkv * G, Hkv, 0, d, W, ratio, [rng.randrange(1, 2500) for _ in range(rng.randrange(2, 5))]
    return rng.choice([1, 2]), Hkv * G, Hkv, rng.randrange(500, 3000), d, W, ratio, None


@pytest.mark.parametrize("seed", range(4))
def test_backward_medium_random_shape(seed):
    """Every gradient element at sizes that span many CTAs of the dQ and dK/dV launches."""
    from tests.test_gpu_backward import close as close_grad, gpu_run

    B, Hq, Hkv, L, d, W, ratio, lens = draw_medium_backward(seed)
    w = workloads.make(B, Hq, Hkv, L, d, W, ratio, seed=seed, seqlens=lens, name=f"bmedium{seed}")
    e = torch.randn(w.q.shape, generator=torch.Generator().manual_seed(seed)).bfloat16()
    dq, dk, dv, dg = gpu_run(w, e)
    ref = oracle.backward(w.q, w.k, w.v, w.g, e, w.W, w.ratio, cu_seqlens=w.cu_seqlens)
    T = w.L if w.cu_seqlens is None else int(w.cu_seqlens[-1])
    what = f"medium backward {seed} {(B, Hq, Hkv, L, d, W, ratio, lens)}"
    close_grad(dq[:, :, :T], ref["dq"][:, :, :T], what + " dq")
    close_grad(dk[:, :, :T], ref["dk"][:, :, :T], what + " dk")
    close_grad(dv[:, :, :T], ref["dv"][:, :, :T], what + " dv")
    if (ref["dg"] != 0).any():
        check_dgate(w, e, dg[:, :T], ref["dg"][:, :T], T, what + " dgate")
