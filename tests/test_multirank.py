"""Multi-rank host logic on the CPU (gloo, world size 2).

The forward pass splits across ranks by whole sequences, or by whole
key/value-head groups, with no exchange on the data path.  These tests check
the assignment (every sequence exactly once, balanced by attention cost; every
head exactly once, in whole groups), the per-rank packing, and that two gloo
ranks each running their own share reproduce the single-process result
element for element (with the fp64 oracle standing in for the GPU kernels, which the CPU
box does not have).  The max / sum reductions used for whole-job timing are
checked on the same two ranks.
"""
import os
import pickle
import socket

import pytest
import torch
import torch.multiprocessing as mp

import oracle
from token_level_dynamic_seq_b200 import multirank, workloads


def test_shard_covers_every_sequence_once():
    lens = [1024, 16384, 7000, 3, 0, 9000, 12000, 512, 4096]
    for world in (1, 2, 3, 4, 8, 16):
        shards = multirank.shard_sequences(lens, world, 2048, 0.25)
        flat = sorted(s for sh in shards for s in sh)
        assert flat == list(range(len(lens)))
        assert all(sh == sorted(sh) for sh in shards)


def test_shard_balance_lpt_bound():
    torch.manual_seed(0)
    lens = torch.randint(1024, 16385, (64,)).tolist()
    costs = [multirank.sequence_cost(n, 2048, 0.25) for n in lens]
    for world in (2, 4, 8):
        shards = multirank.shard_sequences(lens, world, 2048, 0.25)
        loads = [sum(costs[s] for s in sh) for sh in shards]
        # Greedy LPT: the heaviest rank exceeds the mean by at most the largest single job.
        assert max(loads) <= sum(costs) / world + max(costs)


def test_local_pairs_closed_form():
    for n in (0, 1, 5, 100):
        for w in (1, 3, 100, 1000):
            assert multirank.local_pairs(n, w) == sum(min(i + 1, w) for i in range(n))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_path):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = workloads.make(1, 4, 2, 0, 16, 8, 0.25, seed=3, qkv_scale=1.0, seqlens=[40, 7, 0, 65, 23, 31])
        shards = multirank.shard_sequences(w.seqlens, world, w.W, w.ratio)
        mine = shards[rank]
        q, k, v, g, cu, lens = multirank.pack_sequences(w.q, w.k, w.v, w.g, w.cu_seqlens, mine)
        res = oracle.forward(q, k, v, g, w.W, w.ratio, cu_seqlens=cu)
        # per sequence: its rows of every head
        pieces = {}
        off = 0
        for s, n in zip(mine, lens):
            pieces[s] = res["out"][0, :, off:off + n].clone()
            off += n
        gathered = [None] * world
        dist.all_gather_object(gathered, pieces)
        mx = multirank.max_over_ranks(float(rank + 1))
        sm = multirank.sum_over_ranks(float(sum(lens)))
        if rank == 0:
            with open(out_path, "wb") as f:
                pickle.dump({"gathered": gathered, "max": mx, "sum": sm, "shards": shards}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reproduce_single_process(tmp_path):
    out_path = str(tmp_path / "result.pkl")
    mp.spawn(_rank_main, args=(2, _free_port(), out_path), nprocs=2, join=True)
    with open(out_path, "rb") as f:
        r = pickle.load(f)
    w = workloads.make(1, 4, 2, 0, 16, 8, 0.25, seed=3, qkv_scale=1.0, seqlens=[40, 7, 0, 65, 23, 31])
    full = oracle.forward(w.q, w.k, w.v, w.g, w.W, w.ratio, cu_seqlens=w.cu_seqlens)["out"]
    merged = {}
    for part in r["gathered"]:
        merged.update(part)
    assert sorted(merged) == list(range(len(w.seqlens)))
    cu = w.cu_seqlens.tolist()
    for s, rows in merged.items():
        assert torch.equal(rows, full[0, :, cu[s]:cu[s + 1]])
    assert r["max"] == 2.0
    assert r["sum"] == float(sum(w.seqlens))
    assert all(len(sh) > 0 for sh in r["shards"])


def test_shard_heads_whole_groups():
    for Hq, Hkv in ((32, 8), (8, 8), (6, 2), (4, 1)):
        for world in (1, 2, 3, 4, 8):
            shards = multirank.shard_heads(Hq, Hkv, world)
            G = Hq // Hkv
            covered = []
            for h0, h1, hk0, hk1 in shards:
                assert h0 == hk0 * G and h1 == hk1 * G
                covered += list(range(h0, h1))
            assert covered == list(range(Hq))


def _head_rank_main(rank, world, port, out_path):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = workloads.make(1, 8, 4, 45, 16, 9, 0.25, seed=5, qkv_scale=1.0)
        shard = multirank.shard_heads(w.Hq, w.Hkv, world)[rank]
        q, k, v = multirank.head_slice(w.q, w.k, w.v, shard)
        res = oracle.forward(q, k, v, w.g, w.W, w.ratio)
        gathered = [None] * world
        dist.all_gather_object(gathered, (shard, res["out"], res["sel_idx"].tolist()))
        if rank == 0:
            with open(out_path, "wb") as f:
                pickle.dump(gathered, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_head_shards_reproduce_single_process(tmp_path):
    out_path = str(tmp_path / "heads.pkl")
    mp.spawn(_head_rank_main, args=(2, _free_port(), out_path), nprocs=2, join=True)
    with open(out_path, "rb") as f:
        gathered = pickle.load(f)
    w = workloads.make(1, 8, 4, 45, 16, 9, 0.25, seed=5, qkv_scale=1.0)
    full = oracle.forward(w.q, w.k, w.v, w.g, w.W, w.ratio)
    for (h0, h1, _, _), out, sel in gathered:
        assert sel == full["sel_idx"].tolist()  # every rank recomputes the same selection
        assert torch.equal(out, full["out"][:, h0:h1])
