"""Seeded synthetic inputs for the forward pass (no attention arithmetic here).

Both the CUDA path's tests/benchmark and the CPU oracle draw their inputs from
this module, so it holds only random-number recipes and shapes.  Every draw
uses a CPU ``torch.Generator`` so the data do not depend on the device.

Recipe (fixed order per workload): for the packed varlen workload the
sequence lengths first (they fix the token count), then Q, K, V (one head
slab at a time, drawn in fp32, scaled, rounded to bf16 round-to-nearest-even),
then the gate logits, then (varlen only) the burst starts.

Workloads follow the shapes the pages discuss: contexts from 32K to 128K
tokens with about a fifth of the tokens going global ("Learning When to
Attend", "Empirical Validation and System Optimization"; "The Architecture of
Conditional Attention"), a 4096-token local window ("Local-global attention",
Gemma 2 variant) and packed examples masked per example ("Local-global
attention", Implementation sketch notes, "Packed examples (LongT5)").
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int  # fixed length per sequence, or the packed token count T (varlen)
    d: int
    W: int
    ratio: float
    q: torch.Tensor  # bf16 [B, Hq, L, d]
    k: torch.Tensor  # bf16 [B, Hkv, L, d]
    v: torch.Tensor  # bf16 [B, Hkv, L, d]
    g: torch.Tensor  # fp32 [B, L]
    cu_seqlens: torch.Tensor | None = None  # int32 [nseq + 1] (varlen only)
    seqlens: list = field(default_factory=list)
    recipe: str = ""

    @property
    def nseq(self) -> int:
        return len(self.seqlens)

    @property
    def tokens(self) -> int:
        return int(sum(self.seqlens))


def _draw_heads(gen: torch.Generator, B: int, H: int, L: int, d: int, scale: float) -> torch.Tensor:
    out = torch.empty(B, H, L, d, dtype=torch.bfloat16)
    for b in range(B):
        for h in range(H):
            x = torch.randn(L, d, generator=gen, dtype=torch.float32)
            if scale != 1.0:
                x.mul_(scale)
            out[b, h].copy_(x)  # fp32 -> bf16, round to nearest even
    return out


def make(B: int, Hq: int, Hkv: int, L: int, d: int, W: int, ratio: float, *, seed: int = 0,
         qkv_scale: float = 1.0, seqlens: list | None = None, burst_p: float = 0.0,
         burst_len: int = 64, burst_add: float = 3.0, name: str = "custom") -> Workload:
    """Generic seeded workload.

    ``seqlens`` given: packed varlen layout (B must be 1, L is ignored and set
    to the total).  ``burst_p`` > 0: each position starts a run with that
    probability and ``burst_add`` is added once to every token covered by any
    run of ``burst_len`` tokens starting there (runs clip at the sequence end
    and do not stack).
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    cu = None
    if seqlens is not None:
        assert B == 1
        seqlens = [int(x) for x in seqlens]
        L = sum(seqlens)
        cu = torch.zeros(len(seqlens) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(seqlens, dtype=torch.int64), 0).to(torch.int32)
    else:
        seqlens = [L] * B
    q = _draw_heads(gen, B, Hq, L, d, qkv_scale)
    k = _draw_heads(gen, B, Hkv, L, d, qkv_scale)
    v = _draw_heads(gen, B, Hkv, L, d, qkv_scale)
    g = torch.randn(B, L, generator=gen, dtype=torch.float32)
    if burst_p > 0.0:
        starts = torch.rand(B, L, generator=gen, dtype=torch.float32) < burst_p
        covered = torch.zeros(B, L, dtype=torch.bool)
        bounds = [(0, L)] if cu is None else [(int(cu[i]), int(cu[i + 1])) for i in range(len(seqlens))]
        for b in range(B):
            for lo, hi in bounds:
                idx = torch.nonzero(starts[b, lo:hi]).flatten().tolist()
                for s in idx:
                    covered[b, lo + s: min(hi, lo + s + burst_len)] = True
        g = g + covered.to(torch.float32) * burst_add
    return Workload(name=name, B=B, Hq=Hq, Hkv=Hkv, L=L, d=d, W=W, ratio=ratio, q=q, k=k, v=v, g=g,
                    cu_seqlens=cu, seqlens=seqlens)


# Named workloads -----------------------------------------------------------

RATIO_SWEEP_128K = (0.05, 0.1, 0.2, 0.35, 0.5)

CONFIGS = {
    # name: (description, builder kwargs)
    "tiny": dict(B=1, Hq=2, Hkv=2, L=256, d=64, W=32, ratio=0.25, qkv_scale=1.0 / math.sqrt(64)),
    "c4k": dict(B=2, Hq=8, Hkv=8, L=4096, d=128, W=512, ratio=0.2, qkv_scale=128 ** -0.5),
    "c32k": dict(B=1, Hq=32, Hkv=8, L=32768, d=128, W=4096, ratio=0.2, qkv_scale=1.0),
}
# The headline shape at a quarter of the length: inputs still larger than L2,
# small enough for a many-pass profiler capture.
CONFIGS["c8k"] = dict(B=1, Hq=32, Hkv=8, L=8192, d=128, W=4096, ratio=0.2, qkv_scale=1.0)
for _r in RATIO_SWEEP_128K:
    CONFIGS[f"c128k_r{_r:g}"] = dict(B=1, Hq=32, Hkv=8, L=131072, d=128, W=4096, ratio=_r,
                                     qkv_scale=1.0)

VARLEN_NSEQ = 8
VARLEN_MIN, VARLEN_MAX = 1024, 16384


def varlen_seqlens(seed: int = 0) -> list:
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return torch.randint(VARLEN_MIN, VARLEN_MAX + 1, (VARLEN_NSEQ,), generator=gen).tolist()


def describe(name: str) -> str:
    if name == "varlen":
        return ("packed varlen: 8 sequences, lengths U{1024..16384} (seeded), Hq=32, Hkv=8, d=128, "
                "W=2048, ratio=0.25; Q/K/V bf16 N(0,1); gate fp32 N(0,1) + 3.0 on runs of 64 tokens "
                "starting with probability 0.01")
    c = CONFIGS[name]
    return (f"B={c['B']}, Hq={c['Hq']}, Hkv={c['Hkv']}, L={c['L']}, d={c['d']}, W={c['W']}, "
            f"ratio={c['ratio']}; Q/K/V bf16 N(0,1)*{c['qkv_scale']:.4g}; gate fp32 N(0,1)")


def load(name: str, seed: int = 0) -> Workload:
    """Build a named workload: tiny, c4k, c8k, c32k (headline), c128k_r{ratio}, varlen."""
    if name == "varlen":
        # Lengths come from a generator seeded with `seed`; Q, K, V, the gate
        # logits and the burst starts (in that order) from one seeded with seed + 1.
        lens = varlen_seqlens(seed)
        w = make(1, 32, 8, 0, 128, 2048, 0.25, seed=seed + 1, qkv_scale=1.0, seqlens=lens,
                 burst_p=0.01, burst_len=64, burst_add=3.0, name="varlen")
    else:
        c = dict(CONFIGS[name])
        w = make(c.pop("B"), c.pop("Hq"), c.pop("Hkv"), c.pop("L"), c.pop("d"), c.pop("W"),
                 c.pop("ratio"), seed=seed, name=name, **c)
    w.recipe = describe(name)
    return w
