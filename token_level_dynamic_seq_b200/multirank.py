"""Splitting the forward pass across ranks (one process per GPU).

The forward pass partitions into independent problems, two ways:
  * by sequence: the sequences of a batch never attend to one another
    ("Local-global attention", Implementation sketch notes, "Packed examples
    (LongT5)") and the budget is per sequence;
  * by head: every head attends on its own, and the selection depends only on
    the gate logits, which every rank holds whole (they are tiny), so each rank
    runs its key/value-head groups and recomputes the same selection.
Either way no collective touches the attention data.  This module holds the
host logic for both: a longest-processing-time assignment of sequences to
ranks by their attention cost, the packing of a rank's sequences into its own
varlen batch, the split of heads in whole key/value groups, and the max / sum
reductions used to report whole-job timings.
"""
from __future__ import annotations

import heapq

import torch


def num_selected(ratio: float, length: int) -> int:
    """Budget count; the library's own implementation (the C ABI) is authoritative."""
    from token_level_dynamic_seq_b200 import num_selected as _ns
    return _ns(ratio, length)


def local_pairs(n: int, window: int) -> int:
    """sum_{i < n} min(i + 1, W): (query, key) pairs of the windowed branch."""
    w = min(int(window), int(n))
    return w * (w + 1) // 2 + (int(n) - w) * w


def sequence_cost(n: int, window: int, ratio: float) -> float:
    """Attention pairs of one sequence: windowed pairs plus the expected pairs of
    the selected queries (k queries with prefixes averaging (n + 1) / 2 keys)."""
    k = num_selected(ratio, n)
    return float(local_pairs(n, window)) + k * (n + 1) / 2.0


def shard_sequences(seqlens, world: int, window: int, ratio: float) -> list[list[int]]:
    """Assign sequence indices to `world` ranks, longest cost first to the least
    loaded rank.  Every sequence goes to exactly one rank; each rank's list is
    in ascending index order."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(seqlens)), key=lambda s: (-sequence_cost(seqlens[s], window, ratio), s))
    heap = [(0.0, r) for r in range(world)]
    heapq.heapify(heap)
    out = [[] for _ in range(world)]
    for s in order:
        load, r = heapq.heappop(heap)
        out[r].append(s)
        heapq.heappush(heap, (load + sequence_cost(seqlens[s], window, ratio), r))
    return [sorted(x) for x in out]


def pack_sequences(q, k, v, g, cu_seqlens, seq_ids):
    """Gather sequences `seq_ids` of a packed batch ([1, H, T, d] tensors, gate
    [1, T], int32 cu_seqlens) into a packed batch of their own.  Returns
    (q, k, v, g, cu_seqlens, seqlens) for the subset, same device as the input."""
    cu = [int(x) for x in cu_seqlens.tolist()]
    spans = [(cu[s], cu[s + 1]) for s in seq_ids]
    idx = torch.cat([torch.arange(a, b) for a, b in spans]) if spans else torch.zeros(0, dtype=torch.long)
    idx = idx.to(q.device)
    lens = [b - a for a, b in spans]
    sub_cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    if lens:
        sub_cu[1:] = torch.cumsum(torch.tensor(lens, dtype=torch.int64), 0).to(torch.int32)
    return (q.index_select(2, idx).contiguous(), k.index_select(2, idx).contiguous(),
            v.index_select(2, idx).contiguous(), g.index_select(1, idx).contiguous(),
            sub_cu.to(cu_seqlens.device), lens)


def _reduce(value: float, op, device=None) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(value: float, device=None) -> float:
    """Largest value over all ranks (e.g. the slowest rank's time)."""
    import torch.distributed as dist
    return _reduce(value, dist.ReduceOp.MAX, device)


def sum_over_ranks(value: float, device=None) -> float:
    """Sum over all ranks (e.g. tokens processed by the whole job)."""
    import torch.distributed as dist
    return _reduce(value, dist.ReduceOp.SUM, device)


def shard_heads(Hq: int, Hkv: int, world: int) -> list[tuple[int, int, int, int]]:
    """Split the query heads over ranks in whole key/value groups (GQA: query head h
    reads key/value head h / (Hq / Hkv)), so a rank needs only its own K/V heads and no
    exchange on the data path.  Returns per rank (h0, h1, hk0, hk1): query heads
    [h0, h1) and key/value heads [hk0, hk1); ranks beyond Hkv get empty ranges."""
    if world < 1 or Hkv < 1 or Hq % Hkv:
        raise ValueError("need world >= 1 and Hq a multiple of Hkv")
    G = Hq // Hkv
    out = []
    for r in range(world):
        hk0 = (Hkv * r) // world
        hk1 = (Hkv * (r + 1)) // world
        out.append((hk0 * G, hk1 * G, hk0, hk1))
    return out


def head_slice(q, k, v, shard):
    """The rank's share of [B, H, L, d] tensors for one shard from shard_heads."""
    h0, h1, hk0, hk1 = shard
    return q[:, h0:h1].contiguous(), k[:, hk0:hk1].contiguous(), v[:, hk0:hk1].contiguous()
