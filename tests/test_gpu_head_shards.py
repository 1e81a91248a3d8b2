"""Head-sharded forward on the CUDA path.

The forward pass splits across ranks by whole key/value-head groups with no
exchange on the data path: every rank holds the (tiny) gate, recomputes the
same selection and runs its own groups ("LoGo: Token-Level Dynamic
Local-Global Attention", Abstract: one gate decision per token, shared by
the heads).  Here every rank's share, from ``multirank.shard_heads`` and
``multirank.head_slice``, runs through ``logo.forward`` one after another
on the one GPU (each share is an independent launch; nothing waits on
another rank), for 2, 4 and 8 ranks.  Checks: the selection is the same
bits on every share and equals the oracle's; the reassembled output equals
the single-launch output bit for bit and the oracle within the forward's
tolerance (every element on tiny and c4k; at the 32K headline size, rows that
reach every CTA of both launches).
"""
import pytest
import torch

import oracle
import token_level_dynamic_seq_b200 as logo
from token_level_dynamic_seq_b200 import multirank, workloads

from tests.test_gpu_parity import check_every_cta, close, oracle_sel_lists, sel_lists

pytestmark = pytest.mark.gpu


def sharded_forward(w, world):
    """Each rank's share run on its own; returns (reassembled out, per-rank selection lists)."""
    g = w.g.cuda()
    parts, lists = [], []
    for shard in multirank.shard_heads(w.Hq, w.Hkv, world):
        h0, h1, _, _ = shard
        if h1 == h0:
            continue
        q, k, v = (x.cuda() for x in multirank.head_slice(w.q, w.k, w.v, shard))
        out, sel, cu_sel = logo.forward(q, k, v, g, w.W, w.ratio)
        torch.cuda.synchronize()
        parts.append((h0, out))
        lists.append(sel_lists(sel, cu_sel))
        del q, k, v
    out = torch.cat([o for _, o in sorted(parts, key=lambda t: t[0])], dim=1)
    return out, lists


@pytest.mark.parametrize("name", ["tiny", "c4k", "c32k"])
def test_head_shards_match_single_launch_and_oracle(name):
    w = workloads.load(name)
    single, sel, cu_sel = logo.forward(w.q.cuda(), w.k.cuda(), w.v.cuda(), w.g.cuda(), w.W, w.ratio)
    single_lists = sel_lists(sel, cu_sel)
    want_lists = oracle_sel_lists(w)
    assert single_lists == want_lists
    ref = None
    if name != "c32k":
        ref = oracle.forward(w.q, w.k, w.v, w.g, w.W, w.ratio)["out"]
    for world in (2, 4, 8):
        out, lists = sharded_forward(w, world)
        assert all(x == want_lists for x in lists), f"world {world}: a share's selection differs"
        assert torch.equal(out, single), f"world {world}: reassembled heads differ from one launch"
        if ref is not None:
            close(out, ref, f"{name} world {world}")
        elif world == 8:
            # bitwise equal to the single launch for every world; one comparison with the oracle
            check_every_cta(w, out, want_lists, n_inner=0)
        del out
        torch.cuda.empty_cache()
