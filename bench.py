#!/usr/bin/env python
"""Benchmark of the iS-KV hot path on B200: compressed-KV decode over a
32K-token, 36-layer, batch-8 Qwen3-8B-shaped cache (8 KV / 32 query heads,
d 128, r_K 32, r_V 64, W 1024, bf16 K/V and coefficients, fp32 bases).

One bench step = one fold period: 64 decode steps (per layer: append one
token, decode attention for 32 query heads of 8 sequences), then one block
fold of every layer (project, QR, core SVD, basis update, coefficient
resync).  value = decode steps/s (each step = one token for all 8 sequences
through all 36 layers); every timed step contains exactly one fold, so the
block update is amortized honestly.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl iskv|reference]

Multi-GPU: one process per GPU (torchrun), each an independent replica with
its own batch (weak scaling, no data-path collective); rank 0 prints the
max-over-ranks timing.  ``--impl reference`` times the float64 CPU oracle on
the host cores on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import threading
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "compressed-KV decode steps/s at 32K ctx; block-update µs; % of HBM roofline"
UNIT = "decode steps/s"

WORKLOADS = {
    # name: batch, layers, kv_heads, q_heads, rank_k, rank_v, window, prefill, coef
    "qwen3-36L-b8-32k": dict(batch=8, layers=36, kv_heads=8, q_heads=32, rank_k=32, rank_v=64,
                             window=1024, prefill=32768, coef="bf16", gen="qwen3"),
    "qwen3-1L-b8-32k": dict(batch=8, layers=1, kv_heads=8, q_heads=32, rank_k=32, rank_v=64,
                            window=1024, prefill=32768, coef="bf16", gen="qwen3"),
    "qwen3-1L-b1-16k": dict(batch=1, layers=1, kv_heads=8, q_heads=32, rank_k=32, rank_v=64,
                            window=1024, prefill=16384, coef="f32", gen="qwen3"),
    # one factor per sequence over its 8 KV heads (D = 1024) at the explainer's
    # worked-example ranks for Qwen3-8B (r_K 64, r_V 96)
    "qwen3-1L-b8-32k-joint": dict(batch=8, layers=1, kv_heads=8, q_heads=32, rank_k=64,
                                  rank_v=96, window=1024, prefill=32768, coef="bf16",
                                  gen="qwen3", joint=1),
    # one point of the sweep (r 32, 64K, batch 32) as its own workload: the decode
    # runs the query-side RoPE kernel there (>= 200 folded tiles per SM)
    "qwen3-1L-b32-64k-r32": dict(batch=32, layers=1, kv_heads=8, q_heads=32, rank_k=32, rank_v=32,
                                 window=1024, prefill=65536, coef="bf16", gen="qwen3"),
    # low-bit latent-channel codes: K 16 ch x 8 b + 16 x 4 b, V 16 x 8 + 16 x 4 + 32 x 2
    "qwen3-1L-b8-32k-codes": dict(batch=8, layers=1, kv_heads=8, q_heads=32, rank_k=32, rank_v=64,
                                  window=1024, prefill=32768, coef="codes", gen="qwen3",
                                  quant_k=((16, 8), (16, 4)),
                                  quant_v=((16, 8), (16, 4), (32, 2))),
}
# Long chain-of-thought growth: 36 layers, batch 1, grown from 8K to 128K
# tokens; timed at each context bin, 30% of the decode steps carry queries
# aimed at tokens older than 8K (recall of compressed history).
GROWTH = {"cot-128k": dict(batch=1, layers=36, kv_heads=8, q_heads=32, rank_k=64, rank_v=96,
                           window=2048, coef="bf16", gen="cot",
                           bins=[8192, 16384, 32768, 65536, 131072], recall=0.3,
                           recall_age=8192)}
# One-layer sweep: ranks x contexts x batches, r_K = r_V = r, W 1024, plus the
# no-synchronization ablation's reconstruction drift at one point.
SWEEP = {"sweep": dict(layers=1, kv_heads=8, q_heads=32, window=1024, coef="bf16", gen="qwen3",
                       ranks=[16, 32, 64, 128], contexts=[4096, 16384, 65536, 262144],
                       batches=[1, 8, 32])}
DEFAULT_WORKLOAD = "qwen3-36L-b8-32k"
L2_BYTES = 126e6   # B200 L2
D = 128
BLOCK = 64


# DRAM bytes (read + write) of one decode-attention launch of the named kernel
# at a workload's per-layer shape, taken from an ncu capture of the one-layer
# workload (the 36-layer run issues the same launch once per layer).  Not measured by this
# run: reported as copied, with its source, and only while the decode kernel
# is the one that was captured (None otherwise, and for other workloads).
DECODE_TRAFFIC = {("qwen3-36L-b8-32k", "decode_tc_kernel"): 434.3e6,
                  ("qwen3-1L-b8-32k", "decode_tc_kernel"): 434.3e6,
                  ("qwen3-1L-b32-64k-r32", "decode_u_kernel"): 2338.4e6}
DECODE_TRAFFIC_SOURCE = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of one decode launch "
                         "at this per-layer shape (full ncu capture of the decode kernel on the "
                         "one-layer workload of this shape); copied, not measured in this run")



# the library's names of its decode kernels (Cache.decode_kernel) -> kernel symbols
KERNEL_OF = {"cuda_core": "decode_kernel", "rotate": "decode_tc_kernel", "query_rope": "decode_u_kernel"}


KERNEL_TEXT = {
    "decode_u_kernel": "decode_u_kernel (persistent split-K decode attention, RoPE folded into the "
                       "queries: U = position table x (query, basis) products on the tensor cores, "
                       "per-head combine fused), one launch per layer call",
    "decode_tc_kernel": "decode_tc_kernel (persistent split-K decode attention, keys rebuilt and "
                        "rotated per tile, per-head combine fused), one launch per layer call",
    "decode_kernel": "decode_kernel (split-K fp32 CUDA-core decode) + combine_kernel, timed "
                     "together per layer call",
}

# What the path computes in: storage, tensor-core operand and accumulator types.
PRECISION_ROT = ("bf16 K/V and coefficients in HBM, fp32 bases; decode: bf16 MMA rebuilds keys "
                 "(basis as bf16 hi+lo) into fp32, RoPE in fp32, rotated keys rounded to fp16, "
                 "scores by fp16 MMA with fp16 hi+lo queries, p as bf16 hi+lo, fp32 softmax and "
                 "accumulators; rewrite: bf16 MMA with an fp32-exact 3-part split of W_top; "
                 "fold: fp32")
PRECISION_U = ("bf16 K/V and coefficients in HBM, fp32 bases; decode: per tile an fp16 MMA of the "
               "rows' position table (cos, sin rounded to fp16) with the head's query-basis "
               "products (fp32, rounded to fp16), fp32 accumulate; scores as fp32 FMAs of the bf16 "
               "coefficients with those products; exact rows rotated and scored in fp32; p as "
               "bf16 hi+lo for the bf16 value MMA, fp32 softmax and accumulators; rewrite: bf16 MMA "
               "with an fp32-exact 3-part split of W_top; fold: fp32")
PRECISION = {"decode_u_kernel": PRECISION_U, "decode_tc_kernel": PRECISION_ROT,
             "decode_kernel": "stored K/V and coefficients widened to fp32; decode, softmax and "
                              "accumulators in fp32 on the CUDA cores; fold: fp32"}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            j = json.load(fh)
        return float(j["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return 6650.0, "fallback 6.65 TB/s (no MEASURED_PEAKS.json)"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []
        self.first = 0

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def start(self):
        """Start sampling and return once the first sample has arrived (at most
        a few seconds), so that even a short timed region is covered."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        threading.Thread(target=self._read, daemon=True).start()
        t_end = time.time() + 5.0
        while not self.lines and time.time() < t_end and self.proc.poll() is None:
            time.sleep(0.02)
        self.first = len(self.lines)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        # at least one sample taken after the timed region started
        t_end = time.time() + 1.0
        while len(self.lines) <= self.first and time.time() < t_end and self.proc.poll() is None:
            time.sleep(0.02)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        return parse_clock_samples(self.lines[self.first:])


def parse_clock_samples(lines):
    """Median SM clock, max clock and the throttle reasons seen in
    `nvidia-smi --format=csv,noheader,nounits` lines of ClockSampler.Q."""
    sm, smax, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in "".join(lines).strip().splitlines():
        f = [x.strip() for x in line.split(",")]
        if len(f) < 9:
            continue
        try:
            sm.append(float(f[1]))
            smax.append(float(f[2]))
        except ValueError:
            continue
        for n, v in zip(names, f[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(smax) if smax else None,
            "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------


def oracle_sample(wl, budget_s: float = 15.0, seed: int = 0):
    """Time the float64 oracle, as it stands, on a bounded sample of the
    workload: head decodes at the workload's context and block folds; scale
    to decode steps/s of the full workload (all layers, sequences, heads,
    one fold per 64 steps)."""
    import numpy as np
    from oracle import HeadFactor, dense_decode, fold_block

    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    rng = np.random.default_rng(seed)
    T = wl["prefill"]
    n_c = ((T - wl["window"]) // BLOCK) * BLOCK
    g = wl["q_heads"] // wl["kv_heads"]

    def factor(r):
        B, _ = np.linalg.qr(rng.standard_normal((D, r)))
        f = HeadFactor(D, r, wl["window"])
        f.B = B
        f.S = np.sort(rng.uniform(1, 50, r))[::-1]
        f.C = rng.standard_normal((n_c, r))
        f.n_c = n_c
        f.rows = rng.standard_normal((T, D))
        return f

    fk, fv = factor(wl["rank_k"]), factor(wl["rank_v"])
    q = rng.standard_normal((g, D))
    t_dec, n_dec = 0.0, 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s * 0.6 or n_dec < 2:
        a = time.perf_counter()
        dense_decode(q, fk.full(), fv.full(), 1e6)
        t_dec += time.perf_counter() - a
        n_dec += 1
    t_fold, n_fold = 0.0, 0
    t1 = time.perf_counter()
    while time.perf_counter() - t1 < budget_s * 0.4 or n_fold < 2:
        for f in (fk, fv):
            X = rng.standard_normal((BLOCK, D))
            a = time.perf_counter()
            res = fold_block(f.B, f.S, X)
            f.C @ res.W_top                    # step (e) over the history
            t_fold += time.perf_counter() - a
            n_fold += 1
    heads = wl["layers"] * wl["batch"] * wl["kv_heads"]
    per_dec = t_dec / n_dec
    per_fold = t_fold / n_fold                   # one factor (K or V), averaged
    step_s = heads * per_dec + 2 * heads * per_fold / BLOCK
    sample = (f"{n_dec} head-decodes ({g} query heads over {T} tokens) and {n_fold} factor folds "
              f"(with the rewrite of {n_c} rows) at the workload's shapes; scaled to {heads} "
              f"(layer, sequence, KV head) decodes plus 1/64 fold of {2 * heads} factors per step")
    return 1.0 / step_s, cores, sample, t_dec + t_fold


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------


def max_over_ranks(x: float, world: int, device) -> float:
    """Largest value of x over all ranks (the slowest replica sets the time)."""
    if world == 1:
        return x
    import torch
    t = torch.tensor([x], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(ms_max: float, steps: int, world: int) -> float:
    """Whole-job decode steps/s: every rank runs its own replica (own batch),
    so the job completes steps * 64 decode steps per rank in the slowest
    rank's time."""
    return steps * BLOCK * world / (ms_max / 1e3)


def replica_seeds(rank: int):
    """Seeds of the K, V and query streams of one replica (distinct per rank)."""
    return 1000 * rank + 1, 1000 * rank + 2, 1000 * rank + 3


def run_iskv(args, rank, world, local_rank):
    import torch

    import online_rank_kv_b200 as ik
    import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if args.async_update:
        # decode on a high-priority stream, block updates on a low-priority one:
        # the block scheduler then places pending decode CTAs first
        low, high = torch.cuda.Stream.priority_range()
        torch.cuda.set_stream(torch.cuda.Stream(device=dev, priority=high))
    wl = WORKLOADS[args.workload]
    L, Bsz, H, Hq = wl["layers"], wl["batch"], wl["kv_heads"], wl["q_heads"]
    g = Hq // H
    coef = ik.BF16 if wl["coef"] == "bf16" else ik.F32
    codes = wl["coef"] == "codes"
    e2e_periods = max(1, args.steps // 2)
    measure_periods = 1
    periods = args.warmup + args.steps + e2e_periods + measure_periods
    n_steps = periods * BLOCK
    max_tokens = wl["prefill"] + n_steps + BLOCK
    cfg = ik.Config(batch=Bsz, layers=L, kv_heads=H, q_heads=Hq, rank_k=wl["rank_k"],
                    rank_v=wl["rank_v"], window=wl["window"], max_tokens=max_tokens,
                    kv_dtype=ik.BF16, coef_dtype=coef, use_rope=1, rope_theta=1e6,
                    max_deferred=64, protect=args.protect, joint=wl.get("joint", 0),
                    coef_quant=1 if codes else 0, quant_k=wl.get("quant_k", ()),
                    quant_v=wl.get("quant_v", ()))
    cache = ik.Cache(cfg)
    P = args.protect
    kdt = torch.bfloat16
    nh = L * Bsz * H
    seed_k, seed_v, seed_q = replica_seeds(rank)
    ks = synth.KVStream(synth.spec_for(wl["gen"], "K"), nh, seed=seed_k, device=dev, dtype=kdt)
    vs = synth.KVStream(synth.spec_for(wl["gen"], "V"), nh, seed=seed_v, device=dev, dtype=kdt)

    # ---- prefill (untimed): fold with postponed rewrites, one rewrite per 64 folds
    t_pre = time.time()
    folds = 0
    for _ in range(wl["prefill"] // BLOCK):
        k = ks.next(BLOCK).view(L, Bsz, H, BLOCK, D)
        v = vs.next(BLOCK).view(L, Bsz, H, BLOCK, D)
        for l in range(L):
            cache.append(l, k[l], v[l])
        T, n_c = cache.counts(0)
        while (max(0, T - P) - n_c - wl["window"]) // BLOCK >= 1:
            cache.compress_block(ik.ALL_LAYERS, defer=True)
            folds += 1
            if folds % 64 == 0:
                cache.sync(ik.ALL_LAYERS)
            T, n_c = cache.counts(0)
    cache.sync(ik.ALL_LAYERS)
    torch.cuda.synchronize()
    prefill_s = time.time() - t_pre

    # ---- decode inputs for every step, resident in HBM
    kk = ks.next(n_steps).view(L, Bsz, H, n_steps, D).permute(3, 0, 1, 2, 4).contiguous()
    vv = vs.next(n_steps).view(L, Bsz, H, n_steps, D).permute(3, 0, 1, 2, 4).contiguous()
    qq = synth.query_batch(n_steps * L * Bsz * Hq, D, seed=seed_q, device=dev,
                           dtype=kdt).view(n_steps, L, Bsz, Hq, D)
    outs = torch.empty(L, Bsz, Hq, D, dtype=torch.float32, device=dev)
    kk = kk.view(n_steps, L, Bsz, H, 1, D)
    vv = vv.view(n_steps, L, Bsz, H, 1, D)
    stream = torch.cuda.current_stream()

    step_ctr = [0]
    dec_events = []
    step_events = []
    side = (torch.cuda.Stream(device=dev, priority=torch.cuda.Stream.priority_range()[0])
            if args.async_update else None)
    # asynchronous updates: layer l folds at step slot[l] of every 64-step
    # period, on the side stream, right after its decode (its block is ready
    # by then, or one period later; the ring holds up to 64 extra rows)
    slot = [(l * BLOCK) // L for l in range(L)]

    def period(host=None, time_decode=False):
        for s in range(BLOCK):
            i = step_ctr[0]
            step_ctr[0] += 1
            ev = time_decode and (s % 8 == 0)
            if time_decode:
                se = torch.cuda.Event(enable_timing=True)
                se.record(stream)
                step_events.append(se)
            for l in range(L):
                if host is None:
                    cache.append(l, kk[i, l], vv[i, l])
                    if ev:
                        e0 = torch.cuda.Event(enable_timing=True)
                        e1 = torch.cuda.Event(enable_timing=True)
                        e0.record(stream)
                    cache.decode_attention(l, qq[i, l], out=outs[l])
                    if ev:
                        e1.record(stream)
                        T, n_c = cache.counts(l)
                        dec_events.append((e0, e1, T, n_c))
                else:
                    hk, hv, hq, ho = host
                    cache.append(l, hk[i, l], hv[i, l])
                    cache.decode_attention(l, hq[i, l], out=ho[i % 2, l])
                if side is not None and slot[l] == s:
                    T, n_c = cache.counts(l)
                    if (max(0, T - P) - n_c - wl["window"]) // BLOCK >= 1:
                        cache.compress_block_async(l, side, after=stream)
        if side is None:
            cache.compress_block(ik.ALL_LAYERS)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        period()
    barrier()

    clocks = ClockSampler(local_rank)
    clocks.start()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    barrier()
    e_start.record(stream)
    for _ in range(args.steps):
        period(time_decode=True)
    e_end.record(stream)
    step_events.append(e_end)
    barrier()
    clk = clocks.stop()
    ms = max_over_ranks(e_start.elapsed_time(e_end), world, dev)
    per_step_ms = ms / args.steps
    value = job_value(ms, args.steps, world)
    # per-token latency: one decode step of every layer (and whatever block
    # update work lands in it), between consecutive step events
    tok_ms = sorted(step_events[j].elapsed_time(step_events[j + 1])
                    for j in range(len(step_events) - 1))
    token_latency = {"p50_ms": tok_ms[len(tok_ms) // 2], "p99_ms": tok_ms[int(0.99 * (len(tok_ms) - 1))],
                     "max_ms": tok_ms[-1], "steps": len(tok_ms)}

    # decode-attention roofline from the events taken inside the timed region
    peak, peak_src = _peaks()
    dsum, bsum = 0.0, 0.0
    kvb, cb = 2, (2 if coef == ik.BF16 else 4)
    rs = wl["rank_k"] + wl["rank_v"]
    row_bytes = rs * cb   # one coefficient row of K and V
    if codes:
        # codes (bits x channels per group) and one fp32 scale per coded group
        row_bytes = sum(n * b // 8 + (4 if b else 0) for n, b in wl["quant_k"] + wl["quant_v"])
    for e0, e1, T, n_c in dec_events:
        t = e0.elapsed_time(e1) / 1e3
        n_w = T - n_c
        if wl.get("joint"):
            # coefficients once per sequence, bases and exact rows per KV head
            byts = Bsz * n_c * row_bytes + Bsz * H * (2 * n_w * D * kvb + D * rs * 4)
        else:
            byts = Bsz * H * (n_c * row_bytes + 2 * n_w * D * kvb + D * rs * 4)
        byts += Bsz * Hq * D * (kvb + 4)
        dsum += t
        bsum += byts
    dec_avg_us = dsum / max(1, len(dec_events)) * 1e6
    achieved = bsum / dsum / 1e9 if dsum > 0 else 0.0
    step_bytes = bsum / max(1, len(dec_events)) * L   # one decode step over every layer

    # ---- block update timing (fold and rewrite separately), untimed pass
    fold_us = resync_us = None
    if side is not None:
        # bring every layer to the same phase (staggered folds leave up to 63
        # more rows in some rings)
        while True:
            if all((max(0, cache.counts(l)[0] - P) - cache.counts(l)[1] - wl["window"]) // BLOCK < 1
                   for l in range(L)):
                break
            cache.compress_block(ik.ALL_LAYERS)
    for _ in range(BLOCK):
        i = step_ctr[0]
        step_ctr[0] += 1
        for l in range(L):
            cache.append(l, kk[i, l], vv[i, l])
            cache.decode_attention(l, qq[i, l], out=outs[l])
    f0, f1, f2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    cache_T, cache_nc = cache.counts(0)
    f0.record(stream)
    cache.compress_block(ik.ALL_LAYERS, defer=True)
    f1.record(stream)
    cache.sync(ik.ALL_LAYERS)
    f2.record(stream)
    torch.cuda.synchronize()
    fold_us = f0.elapsed_time(f1) * 1e3
    resync_us = f1.elapsed_time(f2) * 1e3
    heads = L * Bsz * H
    resync_bytes = 2 * cache_nc * (wl["rank_k"] + wl["rank_v"]) * cb * heads
    resync_gbs = resync_bytes / (resync_us * 1e-6) / 1e9

    # ---- end to end through the C ABI with pinned host buffers
    hk = kk.cpu().pin_memory()
    hv = vv.cpu().pin_memory()
    hq = qq.cpu().pin_memory()
    ho = torch.empty(2, L, Bsz, Hq, D, dtype=torch.float32).pin_memory()
    barrier()
    x0 = torch.cuda.Event(enable_timing=True)
    x1 = torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for _ in range(e2e_periods):
        period(host=(hk, hv, hq, ho))
    x1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(x0.elapsed_time(x1), world, dev)
    e2e_value = job_value(e2e_ms, e2e_periods, world)
    h2d = BLOCK * L * (2 * Bsz * H * D * kvb + Bsz * Hq * D * kvb)
    d2h = BLOCK * L * Bsz * Hq * D * 4
    status = cache.status()
    kept_bytes, full_bytes = cache.kv_bytes()

    # per decode step and layer: append (K, V) + decode attention (one launch on
    # the tensor-core path; split kernel + combine on the CUDA-core path; coded
    # caches first expand their K and V codes); per period and layer: fold (K, V)
    # + coefficient rewrite (K, V), coded caches also code the new rows (K, V)
    # the decode kernel of the timed calls (the library's choice at the final n_c)
    dec_kernel = KERNEL_OF[cache.decode_kernel(0)]
    per_step = 2 + (1 if coef == ik.BF16 else 3 if codes else 2)
    launches_per_period = L * (BLOCK * per_step + (6 if codes else 4))
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": per_step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "mixed: bf16/fp16 MMA inputs, fp32 accumulate" if coef == ik.BF16 or codes
                 else "fp32 math on bf16 K/V, fp32 coefficients",
        "precision": PRECISION[dec_kernel] if coef == ik.BF16 else "bf16 K/V in HBM, fp32 coefficients "
                     "and bases, fp32 CUDA-core math throughout" if not codes else
                     "bf16 K/V in HBM, coefficients as 8/4/2-bit latent-channel codes with fp32 "
                     "scales per row and group, expanded per call to bf16 tiles (code x scale in "
                     "fp32, rounded to bf16) for the tensor-core decode; " + PRECISION[dec_kernel],
        "data": "synthetic",
        "config": {
            "workload": args.workload, "batch": Bsz, "layers": L, "kv_heads": H, "q_heads": Hq,
            "head_dim": D, "rank_k": wl["rank_k"], "rank_v": wl["rank_v"],
            "window": wl["window"], "context_start": wl["prefill"], "protected_rows": P,
            "storage": f"K/V bf16, coefficients {wl['coef']}, bases fp32",
            "step": "64 decode steps (append + decode attention, every layer) + 1 block fold "
                    "of every layer (fold + coefficient rewrite)",
            "l2": (f"inputs larger than L2 (each decode step streams {step_bytes / 1e9:.2f} GB "
                   f"over {L} layer(s), L2 126 MB)" if step_bytes > L2_BYTES else
                   f"inputs smaller than L2 ({step_bytes / 1e6:.0f} MB per decode step, L2 126 MB): "
                   f"steps reuse L2, no flush"),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        },
        "tokens_per_s": value * Bsz,
        "block_update_mode": "async per layer, staggered over the 64 steps (side stream)"
                             if args.async_update else "sync, all layers at the end of the 64 steps",
        "token_latency": token_latency,
        "block_update_us": fold_us + resync_us,
        "fold_us": fold_us, "resync_us": resync_us, "resync_gbs": resync_gbs,
        "decode_attention_us_avg": dec_avg_us,
        "prefill_s": prefill_s,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": DECODE_TRAFFIC.get((args.workload, dec_kernel))
                     if coef == ik.BF16 and P == 0 and not codes else None,
                     "traffic_source": DECODE_TRAFFIC_SOURCE,
                     "kernel": KERNEL_TEXT[dec_kernel]
                               + ("; the codes are expanded first (expand_codes_kernel, timed "
                                  "inside the call)" if codes else ""),
                     "algorithmic_bytes_per_launch": bsum / max(1, len(dec_events)),
                     "peak_source": peak_src},
        # bytes kept between decode steps at the end of the run against the
        # uncompressed K/V cache of the same length (all layers and heads)
        "persistent_kv": {"bytes": kept_bytes, "full_bytes": full_bytes,
                          "compression": full_bytes / kept_bytes if kept_bytes else None},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_period * args.steps,
        "clocks": clk,
        "device_status": status,
    }
    cache.close()
    return result


def _decode_bytes(Bsz, H, Hq, rK, rV, T, n_c, cb, kvb=2):
    """Algorithmic bytes of one decode call of one layer: coefficients, the
    exact rows (K and V), the bases, queries and outputs."""
    n_w = T - n_c
    per_head = n_c * (rK + rV) * cb + 2 * n_w * D * kvb + D * (rK + rV) * 4
    return Bsz * H * per_head + Bsz * Hq * D * (kvb + 4)


def _time_periods(cache, ik, L, stream, n_periods, inputs, qfn, dec_events, step0):
    """n_periods fold periods: 64 decode steps (append one token, decode, every
    layer), then one fold of every layer with its rewrite.  Decode calls of
    every 8th step are timed with events.  Returns the elapsed ms."""
    import torch
    kk, vv = inputs
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    i = step0
    for _ in range(n_periods):
        for s in range(BLOCK):
            for l in range(L):
                cache.append(l, kk[i, l], vv[i, l])
                q = qfn(i, l)
                if dec_events is not None and s % 8 == 0:
                    a = torch.cuda.Event(enable_timing=True)
                    b = torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    cache.decode_attention(l, q)
                    b.record(stream)
                    T, n_c = cache.counts(l)
                    dec_events.append((a, b, T, n_c))
                else:
                    cache.decode_attention(l, q)
            i += 1
        cache.compress_block(ik.ALL_LAYERS)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def _fold_and_rewrite_us(cache, ik, stream):
    """One fold of every layer with its rewrite postponed, then the rewrite:
    (fold us, rewrite us).  Needs a ready block in every layer."""
    import torch
    f0, f1, f2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    f0.record(stream)
    cache.compress_block(ik.ALL_LAYERS, defer=True)
    f1.record(stream)
    cache.sync(ik.ALL_LAYERS)
    f2.record(stream)
    torch.cuda.synchronize()
    return f0.elapsed_time(f1) * 1e3, f1.elapsed_time(f2) * 1e3


def _prefill_to(cache, ik, ks, vs, L, Bsz, H, W, target, archive=None):
    """Append generated rows until T = target, folding every ready block with
    postponed rewrites (one rewrite per 64 folds).  `archive` (optional)
    receives the pre-RoPE keys at positions 17 mod 512 of every head."""
    folds = 0
    T, _ = cache.counts(0)
    while T < target:
        n = min(512, target - T)
        k = ks.next(n)
        v = vs.next(n)
        if archive is not None:
            for j in range(n):
                if (T + j) % 512 == 17:
                    archive["rows"].append(k[:, j].clone())
                    archive["pos"].append(T + j)
        k = k.view(L, Bsz, H, n, D)
        v = v.view(L, Bsz, H, n, D)
        for l in range(L):
            cache.append(l, k[l], v[l])
        T, n_c = cache.counts(0)
        while (T - n_c - W) // BLOCK >= 1:
            cache.compress_block(ik.ALL_LAYERS, defer=True)
            folds += 1
            if folds % 64 == 0:
                cache.sync(ik.ALL_LAYERS)
            T, n_c = cache.counts(0)
    cache.sync(ik.ALL_LAYERS)


def _bring_to_ready(cache, ik, ks, vs, L, Bsz, H, W):
    """Append rows until every layer has one ready block (for the fold and
    rewrite timing)."""
    T, n_c = cache.counts(0)
    need = W + BLOCK - (T - n_c)
    if need > 0:
        k = ks.next(need).view(L, Bsz, H, need, D)
        v = vs.next(need).view(L, Bsz, H, need, D)
        for l in range(L):
            cache.append(l, k[l], v[l])


def run_growth(args, rank, world, local_rank):
    """Long chain-of-thought decode grown from 8K to 128K tokens: at each
    context bin, `steps` timed fold periods (after one warm-up period), with
    30% of the decode steps aiming every query at a token older than 8K."""
    import torch

    import online_rank_kv_b200 as ik
    import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = GROWTH[args.workload]
    L, Bsz, H, Hq = wl["layers"], wl["batch"], wl["kv_heads"], wl["q_heads"]
    rK, rV, W = wl["rank_k"], wl["rank_v"], wl["window"]
    g = Hq // H
    bins = wl["bins"]
    per_bin = 1 + args.steps
    n_steps = per_bin * BLOCK
    max_tokens = bins[-1] + len(bins) * (n_steps + W + 2 * BLOCK) + 1024
    cfg = ik.Config(batch=Bsz, layers=L, kv_heads=H, q_heads=Hq, rank_k=rK, rank_v=rV, window=W,
                    max_tokens=max_tokens, kv_dtype=ik.BF16, coef_dtype=ik.BF16, use_rope=1,
                    rope_theta=1e6, max_deferred=64, ring_extra=512)
    cache = ik.Cache(cfg)
    nh = L * Bsz * H
    seed_k, seed_v, seed_q = replica_seeds(rank)
    ks = synth.KVStream(synth.spec_for(wl["gen"], "K"), nh, seed=seed_k, device=dev, dtype=torch.bfloat16)
    vs = synth.KVStream(synth.spec_for(wl["gen"], "V"), nh, seed=seed_v, device=dev, dtype=torch.bfloat16)
    archive = {"rows": [], "pos": []}
    stream = torch.cuda.current_stream()
    gq = torch.Generator(device="cpu")
    gq.manual_seed(seed_q)
    peak, peak_src = _peaks()
    clocks = ClockSampler(local_rank)
    clocks.start()
    bins_out = []
    tot_ms, tot_steps = 0.0, 0
    t_pre = 0.0
    for nb in bins:
        a = time.time()
        _prefill_to(cache, ik, ks, vs, L, Bsz, H, W, nb, archive)
        torch.cuda.synchronize()
        t_pre += time.time() - a
        # inputs of this bin's periods, resident in HBM
        kk = ks.next(n_steps).view(L, Bsz, H, n_steps, D).permute(3, 0, 1, 2, 4).contiguous()
        vv = vs.next(n_steps).view(L, Bsz, H, n_steps, D).permute(3, 0, 1, 2, 4).contiguous()
        kk = kk.view(n_steps, L, Bsz, H, 1, D)
        vv = vv.view(n_steps, L, Bsz, H, 1, D)
        qq = synth.query_batch(n_steps * L * Bsz * Hq, D, seed=seed_q + nb, device=dev,
                               dtype=torch.bfloat16).view(n_steps, L, Bsz, Hq, D)
        # recall steps: every query of the step aims at an archived key of its
        # KV head older than recall_age tokens
        T0, _ = cache.counts(0)
        rows = torch.stack(archive["rows"], 1)          # [L*B*H, n_arch, D]
        pos = torch.tensor(archive["pos"])
        old = int((pos < T0 - wl["recall_age"]).sum())
        recall = torch.rand(n_steps, generator=gq) < wl["recall"]
        if old > 0:
            for i in torch.nonzero(recall).flatten().tolist():
                pick = torch.randint(0, old, (L, Bsz, Hq), generator=gq)
                head = (torch.arange(L).view(L, 1, 1) * Bsz + torch.arange(Bsz).view(1, Bsz, 1)) * H \
                    + torch.arange(Hq).view(1, 1, Hq) // g
                kp = rows[head.flatten().to(dev), pick.flatten().to(dev)].double()
                ps = pos[pick.flatten()].to(dev)
                qr = synth.recall_queries(kp, ps, 1e6, 25.0 * D ** 0.5)
                qr = qr / torch.linalg.vector_norm(kp, dim=-1, keepdim=True)
                qq[i] = qr.view(L, Bsz, Hq, D).to(torch.bfloat16)
        dec_events = []
        qfn = lambda i, l: qq[i, l]
        _time_periods(cache, ik, L, stream, 1, (kk, vv), qfn, None, 0)           # warm-up
        ms = _time_periods(cache, ik, L, stream, args.steps, (kk, vv), qfn, dec_events, BLOCK)
        ms = max_over_ranks(ms, world, dev)
        dsum = sum(a.elapsed_time(b) for a, b, _, _ in dec_events) / 1e3
        bsum = sum(_decode_bytes(Bsz, H, Hq, rK, rV, T, n_c, 2) for _, _, T, n_c in dec_events)
        _bring_to_ready(cache, ik, ks, vs, L, Bsz, H, W)
        T1, n_c1 = cache.counts(0)
        fold_us, rw_us = _fold_and_rewrite_us(cache, ik, stream)
        rw_bytes = 2 * n_c1 * (rK + rV) * 2 * L * Bsz * H
        steps = args.steps * BLOCK
        bins_out.append({"context": T0, "decode_kernel": KERNEL_OF[cache.decode_kernel(0)],
                         "steps_per_s": steps / (ms / 1e3) * world,
                         "ms_per_period": ms / args.steps,
                         "decode_us": dsum / max(1, len(dec_events)) * 1e6,
                         "decode_hbm_frac": (bsum / dsum / 1e9) / peak if dsum > 0 else None,
                         "recall_steps": int(recall[BLOCK:].sum()),
                         "fold_us": fold_us, "rewrite_us": rw_us,
                         "rewrite_rows": n_c1, "rewrite_gbs": rw_bytes / (rw_us * 1e-6) / 1e9})
        tot_ms += ms
        tot_steps += steps
        del kk, vv, qq
    clk = clocks.stop()
    status = cache.status()
    kept, full = cache.kv_bytes()
    cache.close()
    value = tot_steps * world / (tot_ms / 1e3)
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": BLOCK, "ms_per_step": tot_ms / (args.steps * len(bins)),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "mixed bf16/fp16 MMA inputs, fp32 accumulate",
        "precision": "; ".join(PRECISION[k] for k in sorted({b["decode_kernel"] for b in bins_out})),
        "data": "synthetic",
        "config": {"workload": args.workload, "batch": Bsz, "layers": L, "kv_heads": H,
                   "q_heads": Hq, "head_dim": D, "rank_k": rK, "rank_v": rV, "window": W,
                   "bins": bins, "recall_fraction": wl["recall"],
                   "recall_age": wl["recall_age"],
                   "step": f"per bin: 1 warm-up + {args.steps} timed fold periods (64 decode "
                           "steps of every layer + 1 fold of every layer with its rewrite)",
                   "l2": "inputs larger than L2 from the 16K bin on (coefficients of 36 layers)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "bins": bins_out,
        "prefill_s": t_pre,
        "persistent_kv": {"bytes": kept, "full_bytes": full,
                          "compression": full / kept if kept else None},
        "peak": {"hbm_gbs": peak, "source": peak_src},
        "gpu_launches": (BLOCK * L * 3 + 4) * args.steps * len(bins),
        "clocks": clk, "device_status": status,
    }


def run_sweep(args, rank, world, local_rank):
    """One-layer sweep over ranks, contexts and batches: one JSON line per
    point (decode steps/s, decode HBM fraction, fold and rewrite time), then
    one line with the no-synchronization ablation's reconstruction drift."""
    import torch

    import online_rank_kv_b200 as ik
    import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = SWEEP[args.workload]
    L, H, Hq, W = wl["layers"], wl["kv_heads"], wl["q_heads"], wl["window"]
    peak, peak_src = _peaks()
    stream = torch.cuda.current_stream()
    seed_k, seed_v, seed_q = replica_seeds(rank)
    periods = max(1, min(args.steps, 2))
    lines = []
    for r in wl["ranks"]:
        for T in wl["contexts"]:
            for Bsz in wl["batches"]:
                n_steps = (1 + periods) * BLOCK
                cfg = ik.Config(batch=Bsz, layers=L, kv_heads=H, q_heads=Hq, rank_k=r, rank_v=r,
                                window=W, max_tokens=T + n_steps + W + 2 * BLOCK + 1024,
                                kv_dtype=ik.BF16, coef_dtype=ik.BF16, use_rope=1, rope_theta=1e6,
                                max_deferred=64, ring_extra=512)
                cache = ik.Cache(cfg)
                nh = L * Bsz * H
                ks = synth.KVStream(synth.spec_for(wl["gen"], "K"), nh, seed=seed_k + r + T, device=dev,
                                    dtype=torch.bfloat16)
                vs = synth.KVStream(synth.spec_for(wl["gen"], "V"), nh, seed=seed_v + r + T, device=dev,
                                    dtype=torch.bfloat16)
                _prefill_to(cache, ik, ks, vs, L, Bsz, H, W, T)
                kk = ks.next(n_steps).view(L, Bsz, H, n_steps, D).permute(3, 0, 1, 2, 4).contiguous()
                vv = vs.next(n_steps).view(L, Bsz, H, n_steps, D).permute(3, 0, 1, 2, 4).contiguous()
                kk = kk.view(n_steps, L, Bsz, H, 1, D)
                vv = vv.view(n_steps, L, Bsz, H, 1, D)
                qq = synth.query_batch(n_steps * L * Bsz * Hq, D, seed=seed_q + r + T + Bsz, device=dev,
                                       dtype=torch.bfloat16).view(n_steps, L, Bsz, Hq, D)
                qfn = lambda i, l: qq[i, l]
                dec_events = []
                clocks = ClockSampler(local_rank)
                clocks.start()
                _time_periods(cache, ik, L, stream, 1, (kk, vv), qfn, None, 0)
                ms = _time_periods(cache, ik, L, stream, periods, (kk, vv), qfn, dec_events, BLOCK)
                clk = clocks.stop()
                ms = max_over_ranks(ms, world, dev)
                dsum = sum(a.elapsed_time(b) for a, b, _, _ in dec_events) / 1e3
                bsum = sum(_decode_bytes(Bsz, H, Hq, r, r, Tn, n_c, 2) for _, _, Tn, n_c in dec_events)
                dk = KERNEL_OF[cache.decode_kernel(0)]   # the kernel the timed calls ran
                _bring_to_ready(cache, ik, ks, vs, L, Bsz, H, W)
                _, n_c1 = cache.counts(0)
                fold_us, rw_us = _fold_and_rewrite_us(cache, ik, stream)
                status = cache.status()
                cache.close()
                del kk, vv, qq, cache, ks, vs
                torch.cuda.empty_cache()
                steps = periods * BLOCK
                line = {
                    "metric": METRIC, "value": steps * world / (ms / 1e3), "unit": UNIT,
                    "n_gpus": world, "steps": periods, "warmup": BLOCK,
                    "ms_per_step": ms / periods, "higher_is_better": True, "scaling": "weak",
                    "vs_baseline": None, "dtype": "mixed bf16/fp16 MMA inputs, fp32 accumulate",
                    "data": "synthetic",
                    "config": {"workload": f"sweep r{r} T{T} B{Bsz}", "batch": Bsz, "layers": L,
                               "kv_heads": H, "q_heads": Hq, "rank_k": r, "rank_v": r, "window": W,
                               "context_start": T,
                               "step": "fold period: 64 decode steps + 1 fold with its rewrite"},
                    "decode_us": dsum / max(1, len(dec_events)) * 1e6,
                    "decode_kernel": dk,
                    "decode_hbm_frac": (bsum / dsum / 1e9) / peak if dsum > 0 else None,
                    "peak": {"hbm_gbs": peak, "source": peak_src},
                    "fold_us": fold_us, "rewrite_us": rw_us,
                    "rewrite_gbs": 2 * n_c1 * 2 * r * 2 * L * Bsz * H / (rw_us * 1e-6) / 1e9,
                    "clocks": clk, "device_status": status,
                }
                lines.append(line)
                if rank == 0:
                    print(json.dumps(line), flush=True)
    # no-synchronization ablation: drift of the rebuilt pre-RoPE keys
    drift = {}
    for sync in (1, 0):
        T = 16384
        cfg = ik.Config(batch=1, layers=1, kv_heads=H, q_heads=Hq, rank_k=32, rank_v=64, window=W,
                        max_tokens=T + 1024, kv_dtype=ik.BF16, coef_dtype=ik.BF16, use_rope=1,
                        rope_theta=1e6, max_deferred=64, ring_extra=512, sync=sync)
        cache = ik.Cache(cfg)
        ks = synth.KVStream(synth.spec_for(wl["gen"], "K"), H, seed=seed_k + 7, device=dev,
                            dtype=torch.bfloat16)
        vs = synth.KVStream(synth.spec_for(wl["gen"], "V"), H, seed=seed_v + 7, device=dev,
                            dtype=torch.bfloat16)
        rows = []
        Tn = 0
        folds = 0
        while Tn < T:
            k = ks.next(512)
            v = vs.next(512)
            rows.append(k.float())
            cache.append(0, k.view(1, H, 512, D), v.view(1, H, 512, D))
            Tn, n_c = cache.counts(0)
            while (Tn - n_c - W) // BLOCK >= 1:
                cache.compress_block(0)
                folds += 1
                Tn, n_c = cache.counts(0)
        Kx = torch.cat(rows, 1)[:, :n_c]
        rec = cache.reconstruct(0, ik.WHICH_K)[0]
        drift[sync] = float(torch.linalg.vector_norm(rec - Kx) / torch.linalg.vector_norm(Kx))
        cache.close()
    if rank == 0:
        print(json.dumps({"metric": "reconstruction drift ||C B^T - K||_F / ||K||_F (pre-RoPE keys)",
                          "workload": "sweep drift r_K 32, T 16384, batch 1, per-fold rewrites",
                          "synchronized": drift[1], "no_sync_ablation": drift[0],
                          "ratio": drift[0] / drift[1] if drift[1] > 0 else None}), flush=True)
    return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=6)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="iskv", choices=["iskv", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(WORKLOADS) + sorted(GROWTH) + sorted(SWEEP))
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--async-update", action="store_true",
                    help="fold each layer on a second stream, one layer per decode step")
    ap.add_argument("--protect", type=int, default=0,
                    help="leading positions kept exact and never folded (protected prompt rows)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        wl = WORKLOADS[args.workload if args.workload in WORKLOADS else DEFAULT_WORKLOAD]
        vals = []
        cores = sample = None
        per = max(2.0, args.cpu_budget / max(1, args.steps + args.warmup))
        for i in range(args.warmup + args.steps):
            v, cores, sample, _ = oracle_sample(wl, budget_s=per, seed=i)
            if i >= args.warmup:
                vals.append(v)
        value = statistics.mean(vals)
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * BLOCK / value, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "batch": wl["batch"], "layers": wl["layers"],
                       "kv_heads": wl["kv_heads"], "q_heads": wl["q_heads"],
                       "context_start": wl["prefill"]},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=180))
    try:
        if args.workload in SWEEP:
            run_sweep(args, rank, world, local_rank)
            return
        if args.workload in GROWTH:
            res = run_growth(args, rank, world, local_rank)
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        res = run_iskv(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                v, cores, sample, used = oracle_sample(WORKLOADS[args.workload],
                                                       budget_s=args.cpu_budget)
                res["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                       "sample": sample + f" ({used:.1f} s of CPU work)"}
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
