"""Benchmark: forward pass of token-level dynamic local-global attention on B200.

Workload (N = 1): B=1, Hq=32, Hkv=8 (GQA), L=32768, d=128, W=4096, ratio 0.2,
bf16 N(0,1) Q/K/V, fp32 N(0,1) gate logits (seeded, synthetic).  One step is
one pass of the whole hot path: selection, local attention, selected-query
global attention with the fused gated merge, launched through the C ABI on one
stream.  With --gpus N (torchrun), every rank runs its own independent
sequence (seed = rank): weak scaling, no collective on the data path; the
timed region is bracketed by barriers and the reported time is the max over
ranks.

Printed: one JSON line (rank 0).  ``--impl reference`` instead times the fp64
CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import random
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

METRIC = "LoGo fwd tokens/s & useful TFLOP/s (frac of bf16 peak) at L=32K, 20% global"
WORKLOAD = "c32k"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-batch", type=int, default=64, help="sequences of the decode workload")
    ap.add_argument("--profile", action="store_true",
                    help="time the kernels only (no end-to-end run, dense comparison or CPU baseline): "
                         "the lean command a profiler capture wraps")
    ap.add_argument("--shard", default="sequences", choices=["sequences", "heads"],
                    help="sequences: each rank runs its own sequence (weak scaling); heads: the ranks split one "
                         "problem by key/value-head groups (strong scaling)")
    return ap.parse_args()


# NVIDIA's datasheet figure for dense bf16 tensor-core throughput of one B200 (the 4.5 PFLOP/s
# they print is with 2:4 sparsity; dense is half).  Reported beside the measured matmul peak.
DATASHEET_DENSE_BF16_TFLOPS = 2250.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), float(p["hbm_gbs"]), "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


def kernel_source_hash():
    import hashlib
    h = hashlib.sha256()
    for name in ("attn.cu", "ptx.cuh", "kernels.cuh"):
        with open(os.path.join(ROOT, "token_level_dynamic_seq_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def decode_source_hash():
    import hashlib
    h = hashlib.sha256()
    for name in ("decode.cu", "ptx.cuh", "kernels.cuh"):
        with open(os.path.join(ROOT, "token_level_dynamic_seq_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def algorithmic_bytes(d, Hq, Hkv, seqlens, counts, last_sel):
    """Bytes each forward kernel must move at least once between HBM and the SMs (bf16 tensors).

    Local launch: Q, K and V read once and O written once: T * d * 2 * (2 Hq + 2 Hkv).
    Global launch, per sequence s with k_s selected tokens, the last at position p_s: the
    selected Q rows (k_s Hq d 2), K and V up to p_s once per key/value head (2 Hkv (p_s + 1) d 2),
    the selected rows of O read (the local branch) and written back (2 k_s Hq d 2), and the gate
    logits and positions of the selected tokens (2 * 4 k_s)."""
    T = sum(seqlens)
    local = T * d * 2 * (2 * Hq + 2 * Hkv)
    glob = 0
    for k_s, p_s in zip(counts, last_sel):
        if k_s > 0:
            glob += k_s * Hq * d * 2 + 2 * Hkv * (p_s + 1) * d * 2 + 2 * k_s * Hq * d * 2 + 8 * k_s
    return {"local": local, "global": glob}


def executed_pairs(G, W, seqlens, cu_sel, sel, tile=128):
    """(query, key) pairs per query head that the forward kernels' MMAs compute, masked ones
    included: every CTA runs its two 128-row query tiles (two heads of one row tile when the
    group size is even, else two consecutive row tiles or chunks of one head) against whole
    128-key tiles from its first key to its last row's position."""
    def ceil(a, b):
        return -(-a // b)
    per_cta = 1 if G % 2 == 0 else 2  # row tiles per head in one CTA
    span = tile * per_cta
    loc = glob = 0
    for s, n in enumerate(seqlens):
        for t0 in range(0, n, span):
            last = min(n, t0 + span) - 1
            loc += per_cta * tile * ceil(last + 1 - max(0, t0 - W + 1), tile) * tile
        k = cu_sel[s + 1] - cu_sel[s]
        for c0 in range(0, k, span):
            last = sel[cu_sel[s] + min(k, c0 + span) - 1]
            glob += per_cta * tile * ceil(last + 1, tile) * tile
    return loc, glob


def dense_causal_comparison(logo, q, k, v, w, ws, stream, dev, peak_burst, ms_step, reps=3):
    """The library's own dense causal attention on the same tensors: the local kernel with the
    window at least every sequence's length, so each query attends to its whole prefix.  Run
    after every other figure is taken; a failure is reported in the line, not raised."""
    try:
        import torch
        ml = max(w.seqlens)
        cu = None if w.cu_seqlens is None else w.cu_seqlens.to(dev)
        tmp = torch.empty_like(q)

        def run():
            logo.local_attn(q, k, v, ml, ws, cu_seqlens=cu, max_seqlen=ml if cu is not None else None, out=tmp,
                            stream=stream)

        run()
        logo.check(ws, stream)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record(stream)
        for _ in range(reps):
            run()
        ev[1].record(stream)
        torch.cuda.synchronize(dev)
        logo.check(ws, stream)
        ms = ev[0].elapsed_time(ev[1]) / reps
        pairs = sum(n * (n + 1) // 2 for n in w.seqlens)  # per head
        flop = 4.0 * q.shape[3] * q.shape[1] * pairs
        tf = flop / (ms * 1e-3) / 1e12
        return {"kernel": "attn_fwd_kernel<d, 0> with W >= every length (dense causal)", "ms": ms,
                "tflops": tf, "frac_of_bf16_peak": tf / peak_burst, "flop": flop,
                "logo_step_over_dense": ms_step / ms}
    except Exception as e:  # reported, never fatal for the bench line
        return {"error": str(e)[:300]}


def threshold_form_timing(logo, g, shape, w, ws, stream, dev, reps=20):
    """The threshold form of the budget rule on the same gate: one controller step (the batch
    target, beta = 1, so the threshold lands on it) and the selection of every position above the
    threshold, each timed alone with CUDA events; a failure is reported in the line."""
    try:
        import torch
        nseq = len(w.seqlens)
        cap = max(w.seqlens)  # a sequence may hold more than its share of the batch's top logits
        tau = torch.zeros(1, dtype=torch.float32, device=dev)
        sel = torch.empty(max(1, nseq * cap), dtype=torch.int32, device=dev)
        cu_sel = torch.empty(nseq + 1, dtype=torch.int32, device=dev)
        target = torch.empty(1, dtype=torch.float32, device=dev)

        def update():
            logo.threshold_update(g, shape, w.ratio, 1.0, tau, ws, target=target, stream=stream)

        def select():
            logo.select_threshold(g, shape, tau, cap, ws, sel, cu_sel, stream=stream)

        out = {}
        for name, fn in (("update_ms", update), ("select_ms", select)):
            for _ in range(3):
                fn()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            ev[0].record(stream)
            for _ in range(reps):
                fn()
            ev[1].record(stream)
            torch.cuda.synchronize(dev)
            out[name] = ev[0].elapsed_time(ev[1]) / reps
        logo.check(ws, stream)
        out["selected"] = int(cu_sel[-1].item())
        return out
    except Exception as e:  # reported, never fatal for the bench line
        return {"error": str(e)[:300]}


def traffic_record():
    """DRAM bytes per launch from the committed ncu summary, if taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return {}
    return rec if rec.get("source_hash") == kernel_source_hash() else {}


def decode_traffic_record():
    """DRAM bytes of one decode step (both kernels) from the committed ncu summary, if taken on
    the current decode source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get("decode", {})
    except Exception:
        return {}
    return rec if rec.get("source_hash") == decode_source_hash() else {}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.samples = []
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
        except Exception:
            uuid = None
        self.uuid = uuid

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 8:
                self.samples.append(parts)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        if not self.samples:
            return None
        sm = []
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        max_mhz = None
        for s in self.samples:
            try:
                sm.append(float(s[0]))
                max_mhz = float(s[1])
            except ValueError:
                continue
            for n, v in zip(names, s[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        busy = [x for x in sm if max_mhz is None or x > 0.3 * max_mhz] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max_mhz, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_baseline(w, seconds_target=15.0, seed=0):
    """The fp64 oracle on a bounded sample of the workload: whole tokens (all heads,
    local branch, global branch where selected, merge), tokens/s on the host cores."""
    import oracle

    sel = set(oracle.select(w.g[0], w.ratio).tolist())
    rng = random.Random(seed)
    n_tok = 2
    elapsed = 0.0
    done = 0
    while elapsed < seconds_target:
        toks = [rng.randrange(w.L) for _ in range(n_tok)]
        seq, head, pos, flag = [], [], [], []
        for t in toks:
            for h in range(w.Hq):
                seq.append(0)
                head.append(h)
                pos.append(t)
                flag.append(int(t in sel))
        t0 = time.perf_counter()
        oracle.rows(w.q, w.k, w.v, w.g, w.W, seq, head, pos, flag)
        elapsed += time.perf_counter() - t0
        done += n_tok
        n_tok = min(64, n_tok * 2)
    cores = oracle.num_threads()
    # the same kind of sample on one thread (a few seconds)
    single = None
    if cores > 1:
        oracle.set_num_threads(1)
        try:
            e1, d1, n1 = 0.0, 0, 1
            while e1 < 3.0:
                toks = [rng.randrange(w.L) for _ in range(n1)]
                seq = [0] * (n1 * w.Hq)
                head = [h for _ in toks for h in range(w.Hq)]
                pos = [t for t in toks for _ in range(w.Hq)]
                flag = [int(t in sel) for t in toks for _ in range(w.Hq)]
                t0 = time.perf_counter()
                oracle.rows(w.q, w.k, w.v, w.g, w.W, seq, head, pos, flag)
                e1 += time.perf_counter() - t0
                d1 += n1
                n1 = min(8, n1 * 2)
            single = {"value": d1 / e1, "unit": "tokens/s", "sample": f"{d1} tokens, {e1:.1f} s"}
        finally:
            oracle.set_num_threads(cores)
    return {"value": done / elapsed, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} random query tokens of the {w.name} workload (all {w.Hq} heads, local + global "
                      f"where selected, merge), {elapsed:.1f} s of fp64 CPU work",
            "single_thread": single}


def run_reference(args, rank, world):
    """The fp64 CPU oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    from token_level_dynamic_seq_b200 import workloads
    import oracle

    w = workloads.load(args.workload, seed=0)
    sel = set(oracle.select(w.g[0], w.ratio).tolist())
    rng = random.Random(1)
    per_step = 8  # tokens per step: a bounded sample of the workload
    times = []
    for it in range(args.warmup + args.steps):
        toks = [rng.randrange(w.L) for _ in range(per_step)]
        seq = [0] * (per_step * w.Hq)
        head = [h for _ in toks for h in range(w.Hq)]
        pos = [t for t in toks for _ in range(w.Hq)]
        flag = [int(t in sel) for t in pos]
        t0 = time.perf_counter()
        oracle.rows(w.q, w.k, w.v, w.g, w.W, seq, head, pos, flag)
        dt = time.perf_counter() - t0
        if it >= args.warmup:
            times.append(dt)
    tot = sum(times)
    value = per_step * len(times) / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * tot / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "desc": w.recipe, "tokens_per_step": per_step},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"{per_step} random query tokens per step (all {w.Hq} heads, local + global "
                                   "where selected, merge)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_decode(args, rank, world):
    """Decode step (row f3): 64 sequences with full 32K caches, W=4096, threshold at the
    controller target for ratio 0.2 over the 64 gate logits; HBM-bound, so the roofline is
    the cache bytes the step must read against the measured HBM bandwidth."""
    import token_level_dynamic_seq_b200 as logo

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    B, Hq, Hkv, L, d, W, ratio = args.decode_batch, 32, 8, 32768, 128, 4096, 0.2
    gen = torch.Generator(device=dev)
    gen.manual_seed(rank)
    q = torch.randn(B, Hq, d, generator=gen, device=dev).to(torch.bfloat16)
    kc = torch.randn(B, Hkv, L, d, generator=gen, device=dev).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, L, d, generator=gen, device=dev).to(torch.bfloat16)
    g = torch.randn(B, generator=gen, device=dev)
    cache_len = torch.full((B,), L, dtype=torch.int32, device=dev)
    shape = logo.Shape(B, Hq, Hkv, L, d, None, B, L)
    ws = logo.decode_workspace(shape, dev)
    tau = torch.zeros(1, dtype=torch.float32, device=dev)
    sws = logo.workspace(logo.Shape(1, 1, 1, B, d, None, 1, B), ratio, dev)
    logo.threshold_update(g.view(1, B), logo.Shape(1, 1, 1, B, d, None, 1, B), ratio, 1.0, tau, sws)
    out = torch.empty_like(q)
    sel = torch.empty(B, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        logo.decode(q, kc, vc, cache_len, g, tau, W, ws=ws, out=out, selected=sel, stream=stream)
    logo.check(ws, stream)
    n_sel = int(sel.sum().item())
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    sampler = ClockSampler(dev.index)
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    ev[0].record(stream)
    for _ in range(args.steps):
        logo.decode(q, kc, vc, cache_len, g, tau, W, ws=ws, out=out, selected=sel, stream=stream)
    ev[1].record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    logo.check(ws, stream)
    ms = ev[0].elapsed_time(ev[1]) / args.steps
    row_bytes = Hkv * d * 2 * 2  # K and V rows of all kv heads at one position
    bytes_step = B * W * row_bytes + n_sel * (L - W) * row_bytes + 2 * B * Hq * d * 2
    peak_burst, peak_sust, hbm, peak_src = peaks()
    achieved = bytes_step / (ms * 1e-3) / 1e9
    line = {
        "metric": f"LoGo decode tokens/s ({B} x 32K caches, W=4096, ~20% global)", "value": B / (ms * 1e-3),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "decode_c32k", "B": B, "Hq": Hq, "Hkv": Hkv, "cache": L, "d": d, "W": W,
                   "ratio": ratio, "selected": n_sel,
                   "l2": f"caches ({kc.numel() * 4 / 1e9:.1f} GB) larger than L2"},
        "roofline": {"kernel": "decode_partial_kernel + decode_combine_kernel", "bound": "hbm",
                     "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": decode_traffic_record().get("bytes_per_step") if B == 64 else None,
                     "peak_source": f"{peak_src} HBM copy bandwidth"},
        "gpu_launches": 2 * args.steps, "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_train(args, rank, world):
    """Training step (row f1): the training forward (selection, local and global branches,
    saving the softmax statistics and both branches of the selected rows) and the backward
    pass (dQ, dK, dV, gate gradient) at 32K tokens, Hq=32, Hkv=8, d=128, W=4096, 20% global.
    Roofline: the backward's useful FLOPs (five matmuls per attended pair, the usual count)
    over its own event-timed duration, against the measured bf16 peak."""
    import token_level_dynamic_seq_b200 as logo
    from token_level_dynamic_seq_b200 import workloads

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    base = args.workload[len("train_"):]
    w = workloads.load(base, seed=rank)
    assert w.cu_seqlens is None, "the training bench takes fixed-length workloads"
    q, k, v, g = w.q.to(dev), w.k.to(dev), w.v.to(dev), w.g.to(dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000 + rank)
    dout = torch.randn(q.shape, generator=gen, device=dev).to(torch.bfloat16)
    stream = torch.cuda.current_stream(dev)
    out, ctx = logo.forward_train(q, k, v, g, w.W, w.ratio, stream=stream)
    dq, dk, dv, dg, bws = logo.backward(q, k, v, g, out, dout, ctx, stream=stream)
    grads = (dq, dk, dv, dg)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        logo.forward_train(q, k, v, g, w.W, w.ratio, ws=ctx["ws"], stream=stream, reuse=(out, ctx))
        if ev is not None:
            ev[1].record(stream)
        logo.backward(q, k, v, g, out, dout, ctx, ws=bws, stream=stream, grads=grads)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    logo.check(ctx["ws"], stream)
    logo.check(bws, stream)
    tot_sel = int(ctx["cu_sel"][-1].item())
    sel_pos = ctx["sel_idx"][:tot_sel].to(torch.int64)
    f_loc, f_glob = logo.useful_flops(w.d, w.Hq, w.seqlens, w.W, sel_pos.tolist())
    fwd_flops = f_loc + f_glob
    bwd_flops = 2.5 * fwd_flops          # dS-recompute-free count: S, dP, dV, dK, dQ per pair
    bwd_exec = 3.5 * fwd_flops           # matmuls this design issues: S and dP twice (dQ and dK/dV kernels)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index)
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    logo.check(ctx["ws"], stream)
    logo.check(bws, stream)
    total_ms = evs[0][0].elapsed_time(evs[-1][2]) / args.steps
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    bwd_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    peak_burst, peak_sust, hbm, peak_src = peaks()
    achieved = bwd_flops / (bwd_ms * 1e-3) / 1e12
    tokens = sum(w.seqlens)
    line = {
        "metric": f"LoGo training step tokens/s (forward + backward, {base})",
        "value": tokens / (total_ms * 1e-3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "d": w.d, "W": w.W,
                   "ratio": w.ratio, "selected": tot_sel,
                   "l2": f"inputs (Q {q.numel() * 2 / 1e6:.0f} MB) " + ("larger" if q.numel() * 2 > 126e6 else "smaller")
                         + " than L2"},
        "forward_ms": fwd_ms, "backward_ms": bwd_ms,
        "backward_useful_tflops": achieved, "backward_executed_tflops": bwd_exec / (bwd_ms * 1e-3) / 1e12,
        "roofline": {"kernel": "backward (prep, dQ selected, dQ local, dK/dV)", "bound": "tensor",
                     "achieved": achieved, "peak": peak_burst, "unit": "TFLOP/s", "frac": achieved / peak_burst,
                     "traffic": None, "peak_source": f"{peak_src} bf16 burst (sustained {peak_sust})"},
        "gpu_launches": 8 * args.steps, "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(args, logo, w, hq, hk, hv, out, ml, dev, stream, world, job_tokens, ws):
    """The same metric end to end through logo_forward_host: page-locked host buffers, the copies
    of Q/K/V/g in and of the output and the selection out inside the timed region."""
    from token_level_dynamic_seq_b200 import multirank

    pin = [x.contiguous().pin_memory() for x in (hq, hk, hv, w.g)]
    cu_host = None if w.cu_seqlens is None else w.cu_seqlens.contiguous().pin_memory()
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    nseq_h = len(w.seqlens)
    sel_host = torch.empty(max(1, nseq_h * logo.num_selected(w.ratio, ml)), dtype=torch.int32).pin_memory()
    cu_sel_host = torch.empty(nseq_h + 1, dtype=torch.int32).pin_memory()
    hbuf = logo.host_buffer(logo.make_shape(pin[0], pin[1], cu_host, ml if cu_host is not None else None),
                            w.ratio, dev, stream)
    h2d = sum(x.numel() * x.element_size() for x in pin) + (0 if cu_host is None else cu_host.numel() * 4)
    d2h = (out_host.numel() * out_host.element_size() + sel_host.numel() * 4 + cu_sel_host.numel() * 4)

    def e2e_step():
        logo.forward_host(*pin, w.W, w.ratio, buf=hbuf, device=dev, cu_seqlens=cu_host,
                          max_seqlen=ml if cu_host is not None else None, out=out_host, sel_idx=sel_host,
                          cu_sel=cu_sel_host, stream=stream)

    e2e_step()  # first call creates the copy streams
    logo.check(hbuf, stream)
    e2e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e2e_ev[0].record(stream)
    n_e2e = max(1, args.e2e_steps)
    for _ in range(n_e2e):
        e2e_step()
    e2e_ev[1].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = multirank.max_over_ranks(e2e_ev[0].elapsed_time(e2e_ev[1]) / n_e2e, device=dev)
    logo.check(ws, stream)
    logo.check(hbuf, stream)

    return {"value": job_tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.workload == "decode_c32k":
        run_decode(args, rank, world)
        return
    if args.workload.startswith("train_"):
        run_train(args, rank, world)
        return
    assert args.warmup >= 3, "at least 3 warm-up steps"

    import token_level_dynamic_seq_b200 as logo
    from token_level_dynamic_seq_b200 import multirank, workloads

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    by_heads = args.shard == "heads"
    w = workloads.load(args.workload, seed=0 if by_heads else rank)
    hq, hk, hv = w.q, w.k, w.v
    if by_heads:
        # every rank holds the whole (tiny) gate and recomputes the same selection
        assert world <= w.Hkv, "head sharding needs at least one key/value head per rank"
        hq, hk, hv = multirank.head_slice(w.q, w.k, w.v, multirank.shard_heads(w.Hq, w.Hkv, world)[rank])
    q, k, v, g = hq.to(dev), hk.to(dev), hv.to(dev), w.g.to(dev)
    Hq_r = q.shape[1]
    cu = None if w.cu_seqlens is None else w.cu_seqlens.to(dev)
    ml = max(w.seqlens)
    shape = logo.make_shape(q, k, cu, ml)
    stream = torch.cuda.current_stream(dev)
    ws = logo.workspace(shape, w.ratio, dev, stream)
    out = torch.empty_like(q)
    cap = max(1, logo.selection_capacity(shape, w.ratio, w.seqlens))
    sel = torch.empty(cap, dtype=torch.int32, device=dev)
    nseq = len(w.seqlens)
    cu_sel = torch.empty(nseq + 1, dtype=torch.int32, device=dev)
    kmax = logo.num_selected(w.ratio, ml)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        logo.select(g, shape, w.ratio, ws, sel, cu_sel, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        logo.local_attn(q, k, v, w.W, ws, cu_seqlens=cu, max_seqlen=ml, out=out, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        logo.global_attn_sparse(q, k, v, g, sel, cu_sel, kmax, out, ws, merge=True, cu_seqlens=cu,
                                max_seqlen=ml, stream=stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    logo.check(ws, stream)

    # useful FLOPs (data-dependent global part from this rank's selection)
    tot_sel = int(cu_sel[-1].item())
    sel_pos_sum = int(sel[:tot_sel].to(torch.int64).sum().item()) + tot_sel
    lp = sum(min(w.W, n) * (min(w.W, n) + 1) // 2 + (n - min(w.W, n)) * min(w.W, n) for n in w.seqlens)
    fl_local = 4 * w.d * Hq_r * lp
    fl_global = 4 * w.d * Hq_r * sel_pos_sum
    tokens = w.tokens
    cu_sel_h = cu_sel.cpu().tolist()
    sel_h = sel[:tot_sel].cpu().tolist()
    last_sel = [sel_h[cu_sel_h[s] + n - 1] if n > 0 else -1
                for s, n in enumerate(cu_sel_h[i + 1] - cu_sel_h[i] for i in range(nseq))]
    ex_loc, ex_glob = executed_pairs(w.Hq // w.Hkv, w.W, w.seqlens, cu_sel_h, sel_h)
    ex_flop = {"local": 4 * w.d * Hq_r * ex_loc, "global": 4 * w.d * Hq_r * ex_glob}
    alg_bytes = algorithmic_bytes(w.d, Hq_r, k.shape[1], w.seqlens, [cu_sel_h[i + 1] - cu_sel_h[i] for i in range(nseq)],
                                  last_sel)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    t_wall0 = time.perf_counter()
    for s in range(args.steps):
        step(evs[s])
    torch.cuda.synchronize(dev)
    t_wall = time.perf_counter() - t_wall0
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    logo.check(ws, stream)

    t_total_ms = evs[0][0].elapsed_time(evs[-1][3])
    per = {"select": [], "local": [], "global": []}
    for e in evs:
        per["select"].append(e[0].elapsed_time(e[1]))
        per["local"].append(e[1].elapsed_time(e[2]))
        per["global"].append(e[2].elapsed_time(e[3]))
    avg = {kk: sum(vv) / len(vv) for kk, vv in per.items()}
    ms_step = multirank.max_over_ranks(t_total_ms / args.steps, device=dev)  # slowest rank
    step_ms = sorted(e[0].elapsed_time(e[3]) for e in evs)
    step_median = multirank.max_over_ranks(statistics.median(step_ms), device=dev)
    step_min = multirank.max_over_ranks(step_ms[0], device=dev)
    # head sharding: all ranks work on the same tokens; sequence sharding: on their own
    job_tokens = tokens if by_heads else int(multirank.sum_over_ranks(tokens, device=dev))

    # end to end through the public API with host buffers: logo_forward_host copies the
    # page-locked inputs in and the output and selection out, inside the timed region
    e2e = run_e2e(args, logo, w, hq, hk, hv, out, ml, dev, stream, world, job_tokens, ws) if not args.profile else None

    peak_burst, peak_sust, hbm, peak_src = peaks()
    dominant = "local" if avg["local"] >= avg["global"] else "global"
    dom_flops = fl_local if dominant == "local" else fl_global
    achieved = dom_flops / (avg[dominant] * 1e-3) / 1e12
    tr = traffic_record() if (w.name == WORKLOAD and world == 1 and not by_heads) else {}
    names = {"local": "attn_fwd_kernel<128, 0>", "global": "attn_fwd_kernel<128, 1>"}
    kern_name = names[dominant]
    traffic_of = {kk: (tr.get(nm, {}).get("bytes_per_launch") if isinstance(tr.get(nm), dict) else None)
                  for kk, nm in names.items()}
    traffic = traffic_of[dominant]
    useful_tflops = multirank.sum_over_ranks(fl_local + fl_global, device=dev) / (ms_step * 1e-3) / 1e12

    line = None
    if rank == 0:
        dense = None if args.profile else dense_causal_comparison(logo, q, k, v, w, ws, stream, dev, peak_burst,
                                                                   ms_step)
        thr = None if args.profile else threshold_form_timing(logo, g, shape, w, ws, stream, dev)
        cpu = None
        if world == 1 and not (args.no_cpu_baseline or args.profile):
            cpu = cpu_baseline(w)
        line = {
            "metric": METRIC,
            "value": job_tokens / (ms_step * 1e-3),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "step_ms_median": step_median,
            "step_ms_min": step_min,
            "higher_is_better": True,
            "scaling": "strong" if by_heads else "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "desc": w.recipe, "tokens_per_rank": tokens,
                       "parallelism": (f"key/value-head groups x{world}" if by_heads
                                       else f"independent sequences x{world}"),
                       "l2": "inputs larger than L2 (Q+K+V+O = %.0f MB > 126 MB)" % (
                           (q.numel() + k.numel() + v.numel() + out.numel()) * 2 / 1e6)},
            "useful_tflops": useful_tflops,
            "useful_frac_of_bf16_peak": useful_tflops / (peak_burst * world),
            "useful_frac_of_datasheet_dense_bf16": useful_tflops / (DATASHEET_DENSE_BF16_TFLOPS * world),
            "kernels_ms": avg,
            "kernels_tflops": {"local": fl_local / (avg["local"] * 1e-3) / 1e12,
                               "global": fl_global / (avg["global"] * 1e-3) / 1e12},
            "useful_flop": {"local": fl_local, "global": fl_global},
            "executed_flop": ex_flop,
            "executed_tflops": {kk: ex_flop[kk] / (avg[kk] * 1e-3) / 1e12 for kk in ("local", "global")},
            "useful_over_executed": {"local": fl_local / ex_flop["local"] if ex_flop["local"] else None,
                                     "global": fl_global / ex_flop["global"] if ex_flop["global"] else None},
            "roofline": {"kernel": kern_name, "bound": "tensor", "achieved": achieved, "peak": peak_burst,
                         "unit": "TFLOP/s", "frac": achieved / peak_burst, "traffic": traffic,
                         "peak_source": f"{peak_src} bf16 burst (sustained {peak_sust})",
                         "frac_of_datasheet_dense_bf16": achieved / DATASHEET_DENSE_BF16_TFLOPS,
                         "datasheet_source": "NVIDIA B200 dense bf16 tensor-core figure, 2.25 PFLOP/s",
                         "algorithmic_bytes": alg_bytes[dominant],
                         "traffic_over_algorithmic": (traffic / alg_bytes[dominant]) if traffic else None},
            "kernels_bytes": {kk: {"algorithmic": alg_bytes[kk], "dram_traffic": traffic_of[kk],
                                   "achieved_gbs": alg_bytes[kk] / (avg[kk] * 1e-3) / 1e9}
                              for kk in ("local", "global")},
            "e2e": e2e,
            "gpu_launches": 3 * args.steps,
            "clocks": clocks,
            "wall_s_timed": t_wall,
            "cpu_baseline": cpu,
            "comparisons": {"dense_causal": dense},
            "threshold_form": thr,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
