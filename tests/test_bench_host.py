"""Host-side logic of bench.py that the GPU run depends on, checked on the CPU with the
library calls and CUDA events replaced by stand-ins: the dense-causal comparison's FLOP
count and its never-fatal error path, and the CPU baseline's single-thread figure."""
import types

import pytest
import torch

import bench
import oracle
from token_level_dynamic_seq_b200 import workloads


class _Event:
    def __init__(self, enable_timing=True):
        pass

    def record(self, stream=None):
        pass

    def elapsed_time(self, other):
        return 6.0  # ms for the whole timed loop


@pytest.fixture
def fake_cuda(monkeypatch):
    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda device=None: None)


def test_dense_causal_comparison_counts_prefix_pairs(fake_cuda):
    calls = []
    lib = types.SimpleNamespace(local_attn=lambda q, k, v, window, ws, **kw: calls.append((window, kw)),
                                check=lambda *a: None)
    w = workloads.make(2, 4, 2, 300, 64, 64, 0.2, seed=0)
    r = bench.dense_causal_comparison(lib, w.q, w.k, w.v, w, None, None, "cpu", 1000.0, ms_step=1.0, reps=3)
    # window = the longest sequence: every query sees its whole prefix
    assert all(c[0] == 300 for c in calls) and len(calls) == 4  # one warm-up + three timed
    pairs = 2 * (300 * 301 // 2)  # two sequences of 300, per head
    assert r["flop"] == pytest.approx(4 * 64 * 4 * pairs)
    assert r["ms"] == pytest.approx(2.0)
    assert r["tflops"] == pytest.approx(r["flop"] / 2e-3 / 1e12)
    assert r["logo_step_over_dense"] == pytest.approx(0.5)


def test_dense_causal_comparison_packed_lengths(fake_cuda):
    lib = types.SimpleNamespace(local_attn=lambda *a, **kw: None, check=lambda *a: None)
    w = workloads.make(1, 4, 2, 0, 64, 64, 0.2, seed=0, seqlens=[10, 20])
    r = bench.dense_causal_comparison(lib, w.q, w.k, w.v, w, None, None, "cpu", 1000.0, ms_step=1.0)
    assert r["flop"] == pytest.approx(4 * 64 * 4 * (55 + 210))


def test_dense_causal_comparison_failure_is_reported_not_raised(fake_cuda):
    def boom(*a, **kw):
        raise RuntimeError("device said no")

    lib = types.SimpleNamespace(local_attn=boom, check=lambda *a: None)
    w = workloads.make(1, 2, 2, 64, 64, 16, 0.2, seed=0)
    r = bench.dense_causal_comparison(lib, w.q, w.k, w.v, w, None, None, "cpu", 1000.0, ms_step=1.0)
    assert "device said no" in r["error"]


def test_cpu_baseline_reports_all_cores_and_one_thread():
    w = workloads.load("tiny")
    before = oracle.num_threads()
    r = bench.cpu_baseline(w, seconds_target=0.5)
    assert r["kind"] == "oracle" and r["value"] > 0 and r["cores"] == before
    assert oracle.num_threads() == before  # restored after the single-thread sample
    if before > 1:
        assert r["single_thread"]["value"] > 0


def _useful_local(L, W):
    return sum(min(i + 1, W) for i in range(L))


def test_executed_pairs_whole_tiles_and_union_for_odd_groups():
    # even group: one 128-row tile per head and CTA; W >= L gives 1 + 2 key tiles for 256 rows
    assert bench.executed_pairs(4, 256, [256], [0, 0], []) == (3 * 128 * 128, 0)
    # odd group: two consecutive row tiles of one head share the union of their key ranges
    loc, glob = bench.executed_pairs(3, 300, [700], [0, 3], [5, 400, 699])
    assert loc == 2 * 128 * 128 * (2 + 4 + 4)
    assert glob == 2 * 128 * 128 * 6  # one pair of chunks reaching position 699
    # never below the useful pairs; equal when every tile is full and unmasked (W = 1 tile)
    for G, W, n in [(2, 4096, 32768), (1, 300, 1000), (4, 1, 129), (5, 17, 300)]:
        loc, _ = bench.executed_pairs(G, W, [n], [0, 0], [])
        assert loc >= _useful_local(n, W)
    loc, _ = bench.executed_pairs(2, 10 ** 6, [512], [0, 0], [])
    assert loc == 128 * 128 * (1 + 2 + 3 + 4)


def test_executed_pairs_packed_sequences_are_independent():
    a = bench.executed_pairs(4, 64, [300], [0, 2], [10, 299])
    b = bench.executed_pairs(4, 64, [1000], [0, 1], [512])
    both = bench.executed_pairs(4, 64, [300, 1000], [0, 2, 3], [10, 299, 512])
    assert both == (a[0] + b[0], a[1] + b[1])
