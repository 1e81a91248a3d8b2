"""The no-allocation variant of the selected-query global branch.

Some callers cannot allocate device memory: a layer that only receives the
op's own tensors from a framework whose allocator owns the device, or a
serving loop where cudaMalloc / cudaFree would synchronise the device.  For
them the library offers logo_global_attn_sparse_noalloc, which takes the same
inputs and outputs but keeps its scratch in a fixed array inside the library.
This test checks, through the C ABI, that it gives the same output as the
workspace entry point, on two calls in a row (the second call must not be
disturbed by what the first left in the shared array).  The file is named so
that pytest collects it last.
"""
import pytest
import torch

import token_level_dynamic_seq_b200 as logo
from token_level_dynamic_seq_b200 import workloads

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3


def close(got, ref):
    got, ref = got.double(), ref.double()
    err = (got - ref).abs().max().item()
    rel = ((got - ref).norm() / ref.norm().clamp_min(1e-30)).item()
    assert torch.isfinite(got).all()
    assert err <= MAX_ABS and rel <= REL_L2, f"max-abs {err:.3e}, rel-L2 {rel:.3e}"


def _case(name, B, Hq, Hkv, L, d, W, ratio, seqlens=None, seed=0):
    w = workloads.make(B, Hq, Hkv, L, d, W, ratio, seed=seed, qkv_scale=1.0, seqlens=seqlens, name=name)
    q, k, v, g = w.q.cuda(), w.k.cuda(), w.v.cuda(), w.g.cuda()
    cu = None if w.cu_seqlens is None else w.cu_seqlens.cuda()
    ml = max(w.seqlens)
    shape = logo.make_shape(q, k, cu, ml)
    ws = logo.workspace(shape, ratio, q.device)
    sel, cu_sel = logo.select(g, shape, ratio, ws)
    local = logo.local_attn(q, k, v, W, ws, cu_seqlens=cu, max_seqlen=ml)
    kmax = logo.num_selected(ratio, ml)
    ref = local.clone()
    logo.global_attn_sparse(q, k, v, g, sel, cu_sel, kmax, ref, ws, merge=True, cu_seqlens=cu, max_seqlen=ml)
    logo.check(ws)
    return dict(q=q, k=k, v=v, g=g, cu=cu, ml=ml, sel=sel, cu_sel=cu_sel, kmax=kmax, local=local, ref=ref)


def _noalloc(c):
    out = c["local"].clone()
    logo.global_attn_sparse_noalloc(c["q"], c["k"], c["v"], c["g"], c["sel"], c["cu_sel"], c["kmax"], out,
                                    merge=True, cu_seqlens=c["cu"], max_seqlen=c["ml"])
    torch.cuda.synchronize()
    return out


def test_noalloc_matches_workspace_entry_point_twice():
    a = _case("gqa", 1, 8, 2, 1500, 128, 700, 0.2)
    b = _case("varlen", 1, 4, 2, 0, 64, 300, 0.35, seqlens=[513, 3, 1024, 129], seed=1)
    for c in (a, b, a):  # two calls in a row on each shape, alternating shapes
        close(_noalloc(c), c["ref"])
        close(_noalloc(c), c["ref"])


def test_noalloc_rejects_bad_shape_without_launching():
    c = _case("tiny", 1, 2, 2, 256, 64, 32, 0.25)
    bad = torch.empty(1, 2, 256, 96, dtype=torch.bfloat16, device="cuda")  # d = 96 is not supported
    with pytest.raises(logo.LogoError):
        logo.global_attn_sparse_noalloc(bad, bad, bad, c["g"], c["sel"], c["cu_sel"], c["kmax"], bad.clone())
