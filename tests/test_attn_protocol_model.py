"""CPU model of the forward kernel's barrier protocol, run on random schedules (race detection).

One CTA of attn_fwd_kernel as agents that run in random interleavings:
  * the TMA thread (Q tiles, then the K/V slot transactions: K(0) alone into slot 1, then
    the pairs (K(j+1), V(j)) into slot j % 2, each after the slot's previous use was released);
  * the copy engine, which lands a started transaction some time later (complete_tx);
  * the MMA-issuing thread (S_i = Q_i K^T and O_i += P_i V, commits);
  * the tensor pipe, which executes issued MMAs and commits strictly in issue order;
  * the two softmax warpgroups (read S_i, maybe rescale O_i, write P_i over S_i, publish;
    at the end read O_i).
Barriers follow mbarrier semantics: a wait on parity P returns once the barrier has completed a
phase whose parity is P (completed phases c: (c & 1) != P).  Every buffer carries a tag of what
it holds; each read checks the tag it needs and each write checks that no reader still needs
the old contents.  A schedule fails on a tag mismatch or a deadlock.  Planted mistakes in the
protocol (a missing wait, a wrong parity, a release committed too early, the rescale after the
publish) must each fail on some schedule, so the model checks something.
"""
import random

import pytest


class Deadlock(Exception):
    pass


WAIT = "wait"  # what an agent yields while a barrier it needs has not completed


class Violation(Exception):
    pass


class Barrier:
    def __init__(self, count):
        self.count, self.pending, self.tx, self.completed = count, count, 0, 0

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, "more arrivals than the barrier's count"
        self._maybe_complete()

    def expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._maybe_complete()

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count

    def done(self, parity):
        return (self.completed & 1) != parity


def run_cta(n_kv, rng, mut=frozenset()):
    """One CTA with n_kv key/value tiles and two query tiles; raises on a violation or deadlock."""
    NQ, SLOTS = 2, 2
    bar = {"q_full": Barrier(1), "o_full": Barrier(1), "drain": Barrier(1)}
    for s in range(SLOTS):
        bar[f"kv_full{s}"] = Barrier(1)
        bar[f"kv_empty{s}"] = Barrier(1)
    for i in range(NQ):
        bar[f"s_full{i}"] = Barrier(1)
        bar[f"p_full{i}"] = Barrier(128)
    # buffers: shared-memory K/V slots, TMEM S/P regions and O accumulators
    kslot = [None] * SLOTS          # tag of the K tile the slot holds
    vslot = [None] * SLOTS
    kslot_readers = [0] * SLOTS     # issued MMAs that will still read the slot
    vslot_readers = [0] * SLOTS
    q_loaded = False
    s_tile = [None] * NQ            # ("S", j) or ("P", j)
    s_unread = [False] * NQ         # an S the softmax has not read yet
    o_acc = [[] for _ in range(NQ)]  # the PV steps accumulated so far
    o_pending = [0] * NQ            # PV MMAs issued but not executed
    engine = []                     # started copies: (slot, kind, tag, barrier, bytes)
    pipe = []                       # issued tensor ops in order
    done_softmax = [False] * NQ

    def tma():
        nonlocal q_loaded
        bar["q_full"].expect_tx(2)
        engine.append(("q", None, None, "q_full", 2))
        # K(0) alone into slot 1
        bar["kv_full1"].expect_tx(1)
        engine.append(("k", 1, 0, "kv_full1", 1))
        uses = [0, 1]  # slot 1 already used once
        for j in range(n_kv):
            sl = j & 1
            use = uses[sl]
            if use >= 1 and "tma_no_empty_wait" not in mut:
                while not bar[f"kv_empty{sl}"].done((use - 1) & 1):
                    yield WAIT
            with_k = j + 1 < n_kv
            bar[f"kv_full{sl}"].expect_tx(2 if with_k else 1)
            engine.append(("v", sl, j, f"kv_full{sl}", 1))
            if with_k:
                engine.append(("k", sl, j + 1, f"kv_full{sl}", 1))
            uses[sl] += 1
            yield

    def copy_engine():
        nonlocal q_loaded
        while True:
            if engine:
                idx = rng.randrange(len(engine))
                kind, sl, tag, b, nbytes = engine.pop(idx)
                if kind == "q":
                    q_loaded = True
                elif kind == "k":
                    if kslot_readers[sl]:
                        raise Violation(f"K({tag}) lands in slot {sl} while MMAs still read K{kslot[sl]}")
                    kslot[sl] = tag
                else:
                    if vslot_readers[sl]:
                        raise Violation(f"V({tag}) lands in slot {sl} while MMAs still read V{vslot[sl]}")
                    vslot[sl] = tag
                bar[b].complete_tx(nbytes)
            yield

    def issue(op):
        kind = op[0]
        if kind == "S":
            _, i, sl, j = op
            kslot_readers[sl] += 1
        elif kind == "PV":
            _, i, sl, j = op
            vslot_readers[sl] += 1
            o_pending[i] += 1
        pipe.append(op)

    def tensor_pipe():
        while True:
            if pipe:
                op = pipe.pop(0)
                kind = op[0]
                if kind == "S":
                    _, i, sl, j = op
                    if not q_loaded:
                        raise Violation("S before Q landed")
                    if kslot[sl] != j:
                        raise Violation(f"S_{i}({j}) reads K{kslot[sl]} from slot {sl}")
                    if s_unread[i] or (s_tile[i] is not None and s_tile[i][0] == "P" and s_tile[i][1] != j - 1):
                        raise Violation(f"S_{i}({j}) overwrites {s_tile[i]}")
                    if s_tile[i] is not None and s_tile[i][0] == "P" and ("PV", i, s_tile[i][1]) not in consumed:
                        raise Violation(f"S_{i}({j}) overwrites P_{i}({s_tile[i][1]}) before PV read it")
                    s_tile[i] = ("S", j)
                    s_unread[i] = True
                    kslot_readers[sl] -= 1
                elif kind == "PV":
                    _, i, sl, j = op
                    if s_tile[i] != ("P", j):
                        raise Violation(f"PV_{i}({j}) reads {s_tile[i]}")
                    if vslot[sl] != j:
                        raise Violation(f"PV_{i}({j}) reads V{vslot[sl]}")
                    if o_acc[i] != list(range(j)) and j > 0:
                        raise Violation(f"PV_{i}({j}) accumulates onto {o_acc[i]}")
                    o_acc[i] = list(range(j + 1)) if j > 0 else [0]
                    consumed.add(("PV", i, j))
                    vslot_readers[sl] -= 1
                    o_pending[i] -= 1
                else:  # commit
                    bar[op[1]].arrive()
            yield

    consumed = set()

    def mma():
        while not bar["q_full"].done(0):
            yield WAIT
        while not bar["kv_full1"].done(0):
            yield WAIT
        for i in range(NQ):
            issue(("S", i, 1, 0))
            issue(("commit", f"s_full{i}"))
        issue(("commit", "kv_empty1"))
        yield
        uses = [0, 1]
        for j in range(n_kv):
            sl = j & 1
            parity = uses[sl] & 1
            if "mma_kv_wrong_parity" in mut:
                parity ^= 1
            while not bar[f"kv_full{sl}"].done(parity):
                yield WAIT
            uses[sl] += 1
            for i in range(NQ):
                if "mma_no_p_wait" not in mut:
                    while not bar[f"p_full{i}"].done(j & 1):
                        yield WAIT
                if "release_before_pv" in mut and i == 0:
                    issue(("commit", f"kv_empty{sl}"))
                issue(("PV", i, sl, j))
                if j + 1 < n_kv:
                    issue(("S", i, sl, j + 1))
                    issue(("commit", f"s_full{i}"))
                yield
            if "release_before_pv" not in mut:
                issue(("commit", f"kv_empty{sl}"))
        issue(("commit", "o_full"))
        issue(("commit", "drain"))
        while not bar["drain"].done(0):
            yield WAIT

    def softmax(i):
        for j in range(n_kv):
            while not bar[f"s_full{i}"].done(j & 1):
                yield WAIT
            if s_tile[i] != ("S", j):
                raise Violation(f"softmax {i} step {j} reads {s_tile[i]}")
            s_unread[i] = False
            yield
            need_rescale = rng.random() < 0.3 and j > 0

            def rescale():
                if o_pending[i]:
                    raise Violation(f"rescale of O_{i} at step {j} while a PV is in flight")
                if o_acc[i] != list(range(j)):
                    raise Violation(f"rescale of O_{i} at step {j} sees {o_acc[i]}")

            if need_rescale and "rescale_after_publish" not in mut:
                rescale()
            s_tile[i] = ("P", j)
            yield
            bar[f"p_full{i}"].arrive(128)
            if need_rescale and "rescale_after_publish" in mut:
                yield
                rescale()
        while not bar["o_full"].done(0):
            yield WAIT
        if o_acc[i] != list(range(n_kv)) or o_pending[i]:
            raise Violation(f"epilogue {i} reads O holding {o_acc[i]}")
        done_softmax[i] = True

    agents = {"tma": tma(), "mma": mma(), "sm0": softmax(0), "sm1": softmax(1)}
    engine_agent, pipe_agent = copy_engine(), tensor_pipe()
    idle = 0
    while agents:
        names = list(agents) + (["engine"] if engine else []) + (["pipe"] if pipe else [])
        g = rng.choice(names)
        if g == "engine":
            next(engine_agent)
            idle = 0
            continue
        if g == "pipe":
            next(pipe_agent)
            idle = 0
            continue
        try:
            r = next(agents[g])
        except StopIteration:
            del agents[g]
            idle = 0
            continue
        idle = idle + 1 if r is WAIT else 0
        if idle > 5000:
            raise Deadlock(f"no progress; agents left {list(agents)}")
    if not all(done_softmax):
        raise Violation("a softmax warpgroup did not finish")


@pytest.mark.parametrize("seed", range(200))
def test_protocol_holds_on_random_schedules(seed):
    rng = random.Random(seed)
    run_cta(rng.randrange(1, 7), rng)


MUTANTS = ["tma_no_empty_wait", "mma_no_p_wait", "mma_kv_wrong_parity", "release_before_pv",
           "rescale_after_publish"]


@pytest.mark.parametrize("mutant", MUTANTS)
def test_planted_protocol_mistakes_are_caught(mutant):
    caught = 0
    for seed in range(300):
        rng = random.Random(seed)
        try:
            run_cta(rng.randrange(2, 7), rng, mut=frozenset([mutant]))
        except (Violation, Deadlock, AssertionError):
            caught += 1
    assert caught > 0, f"no schedule exposed the planted mistake {mutant}"
