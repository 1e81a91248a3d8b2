"""Decode step on the GPU against the fp64 oracle.

One new query per sequence at the end of its key/value cache: local window
always, whole-cache global branch only when the gate passes the threshold.
The selection must match bit for bit; outputs within max-abs 2e-2 and
relative-L2 5e-3 of the oracle.
"""
import pytest
import torch

import oracle
import token_level_dynamic_seq_b200 as logo

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3


def close(got, ref, what):
    got = got.double().cpu()
    err = (got - ref).abs().max().item()
    rel = ((got - ref).norm() / ref.norm().clamp_min(1e-30)).item()
    assert torch.isfinite(got).all(), what
    assert err <= MAX_ABS and rel <= REL_L2, f"{what}: max-abs {err:.3e} rel-L2 {rel:.3e}"


def make_case(B, Hq, Hkv, Lmax, d, lens, seed):
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, d, generator=gen).bfloat16()
    k = torch.randn(B, Hkv, Lmax, d, generator=gen).bfloat16()
    v = torch.randn(B, Hkv, Lmax, d, generator=gen).bfloat16()
    g = torch.randn(B, generator=gen)
    return q, k, v, torch.tensor(lens, dtype=torch.int32), g


CASES = [
    # B, Hq, Hkv, Lmax, d, W, cache lengths
    (8, 8, 2, 3000, 128, 100, [1, 5, 511, 512, 513, 2999, 3000, 0]),
    (6, 4, 4, 1500, 64, 1, [1500, 7, 1024, 1025, 3, 600]),
    (5, 16, 2, 2048, 128, 4096, [2048, 1, 100, 1536, 2000]),
    (4, 2, 1, 700, 128, 256, [700, 256, 257, 2]),
]


@pytest.mark.parametrize("case", CASES)
def test_decode_small_full(case):
    B, Hq, Hkv, Lmax, d, W, lens = case
    q, k, v, cl, g = make_case(B, Hq, Hkv, Lmax, d, lens, seed=sum(lens))
    tau = 0.0
    out, sel = logo.decode(q.cuda(), k.cuda(), v.cuda(), cl.cuda(), g.cuda(),
                           torch.tensor([tau], device="cuda"), W)
    torch.cuda.synchronize()
    ref, _, _, ref_sel = oracle.decode(q, k, v, cl, g, tau, W)
    assert sel.cpu().tolist() == ref_sel.tolist()
    close(out, ref, f"decode {case}")


def test_decode_headline_cache():
    # 8 sequences with 32K caches, Hq=32, Hkv=8, d=128, W=4096; threshold at the
    # controller target for ratio 0.5 over the 8 gate logits.
    B, Hq, Hkv, Lmax, d, W = 8, 32, 8, 32768, 128, 4096
    lens = [32768, 32767, 30001, 4096, 4097, 20000, 1, 32000]
    q, k, v, cl, g = make_case(B, Hq, Hkv, Lmax, d, lens, seed=11)
    tau = oracle.threshold_target(g, 0.5)
    ws = logo.decode_workspace(logo.Shape(B, Hq, Hkv, Lmax, d, None, B, Lmax), "cuda")
    out, sel = logo.decode(q.cuda(), k.cuda(), v.cuda(), cl.cuda(), g.cuda(),
                           torch.tensor([tau], device="cuda"), W, ws=ws)
    logo.check(ws)
    ref, _, _, ref_sel = oracle.decode(q, k, v, cl, g, tau, W)
    assert sel.cpu().tolist() == ref_sel.tolist()
    assert sum(ref_sel.tolist()) == 4
    close(out, ref, "decode 32K caches")


def test_decode_cache_length_beyond_capacity_is_reported():
    q, k, v, cl, g = make_case(2, 4, 2, 64, 64, [64, 65], seed=1)
    ws = logo.decode_workspace(logo.Shape(2, 4, 2, 64, 64, None, 2, 64), "cuda")
    out, sel = logo.decode(q.cuda(), k.cuda(), v.cuda(), cl.cuda(), g.cuda(), torch.tensor([0.0], device="cuda"),
                           16, ws=ws)
    with pytest.raises(logo.LogoError) as e:
        logo.check(ws)
    assert e.value.status == 1
    assert (out[1].float() == 0).all()
    ref, _, _, _ = oracle.decode(q[:1], k[:1], v[:1], cl[:1], g[:1], 0.0, 16)
    close(out[:1], ref, "valid sequence beside an invalid one")
