#!/usr/bin/env python
"""Benchmark of one draft-tree verification step on B200.

A step is the whole hot path over one batch of synthetic input already resident in HBM:
tree-masked attention (one layer) -> LM head + acceptance walk -> KV compaction (one layer).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl etree|reference]

Prints ONE JSON line (rank 0).  `value` is accepted tokens/s over all ranks (sum of a_r + 1 per
request per step), device-timed with CUDA events, max over ranks.  L2 is flushed (a 512 MiB
write, then a 256 MiB read that writes the dirty lines back) before every timed step, outside
the per-call events.  `e2e` repeats the measurement
through the same C-ABI calls with the step's inputs copied from pinned host memory and the
accept results copied back inside the timed region.  `--impl reference` times the fp64 CPU
oracle on the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("tree-verify µs/step & accepted tokens/s at B=1/64/512; "
          "HBM GB/s & TC util vs peak")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- algorithmic work
def attn_work(wl):
    """Algorithmic bytes (KV cache read once, tree K/V, Q in, O out) and FLOPs of one layer."""
    D = wl.head_dim
    kv = 2 * int(wl.kv_len.sum()) * wl.hkv * D * 2
    tree = 2 * wl.n_total * wl.hkv * D * 2
    qo = 2 * wl.n_total * wl.hq * D * 2
    anc = 0
    for r in range(wl.B):
        a0, a1 = int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])
        depth = np.zeros(a1 - a0, dtype=np.int64)
        for i in range(1, a1 - a0):
            depth[i] = depth[wl.parent[a0 + i]] + 1
        anc += int((depth + 1).sum())
    keys = sum(int(wl.kv_len[r]) * wl.nodes(r) for r in range(wl.B)) + anc
    flops = 4 * wl.hq * D * keys
    return kv + tree + qo, flops


def lmhead_work(wl):
    return wl.vocab * wl.hidden_dim * 2 + wl.n_total * wl.hidden_dim * 2, \
        2 * wl.n_total * wl.vocab * wl.hidden_dim


def compact_work(wl, accept_len, n_layers=1):
    return 2 * 2 * int((accept_len + 1).sum()) * wl.hkv * wl.head_dim * 2 * n_layers


def strip_comments(src: str) -> str:
    """C++ source without comments and with runs of whitespace collapsed (string and character
    literals kept), so that a comment edit does not count as a change of the kernel."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":                                  # literal: copy through its closing quote
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "draft_tree_verification_masked_b200", "csrc", n)) as f:
            h.update(strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


# The sources a kernel's DRAM traffic depends on (the traffic entries record their hash).
KERNEL_SOURCES = {"attn": ("attn_tc.cu", "common.cuh", "kernels.cuh"),
                  "lmhead": ("lmhead.cu", "race.cuh", "philox.cuh", "common.cuh", "kernels.cuh"),
                  "compact": ("compact.cu", "common.cuh", "kernels.cuh")}


def kernel_source_hash(kernel: str) -> str:
    return source_hash(*KERNEL_SOURCES[kernel])


def ncu_traffic(kernel: str, workload: str, src_hash: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[f"{kernel}@{workload}"]
        return e["bytes_per_launch"] if e.get("source_hash") == src_hash else None
    except Exception:
        return None


# ----------------------------------------------------------------------------- multi-rank
def reduce_over_ranks(step_s: float, e2e_s: float, tokens: int, world: int, device: str):
    """Whole-job figures: the slowest rank's device times and the sum of accepted tokens."""
    if world <= 1:
        return step_s, e2e_s, float(tokens)
    import torch.distributed as dist
    v = torch.tensor([step_s, e2e_s, float(tokens)], device=device, dtype=torch.float64)
    mx = v.clone()
    dist.all_reduce(mx, op=dist.ReduceOp.MAX)
    dist.all_reduce(v, op=dist.ReduceOp.SUM)
    return float(mx[0]), float(mx[1]), float(v[2])


# ------------------------------------------------------------------------------------ timing
class L2Flush:
    """Evicts the step's data from L2 between timed steps: writes 512 MiB (4x the 126 MB L2),
    then reads a separate 256 MiB so that the dirty lines of that write are written back here,
    outside the timed region, instead of inside the next step."""

    def __init__(self):
        self.wbuf = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
        self.rbuf = torch.ones(64 << 20, dtype=torch.int32, device="cuda")
        self.sink = torch.empty((), dtype=torch.int64, device="cuda")

    def __call__(self):
        self.wbuf.zero_()
        torch.sum(self.rbuf, dim=0, dtype=torch.int64, out=self.sink)


def time_steps(dev, steps, warmup, flush):
    """Whole steps timed with events around the step only (the calls run back to back, as a
    serving loop issues them), then a second pass with events between the three calls for the
    per-call breakdown."""
    for _ in range(warmup):
        dev.step()
    torch.cuda.synchronize()
    whole = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    for i in range(steps):
        flush()
        whole[i][0].record()
        dev.attn()
        dev.lmhead()
        dev.compact()
        whole[i][1].record()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        flush()
        e = ev[i]
        e[0].record()
        dev.attn()
        e[1].record()
        dev.lmhead()
        e[2].record()
        dev.compact()
        e[3].record()
    torch.cuda.synchronize()
    attn = [e[0].elapsed_time(e[1]) for e in ev]
    lm = [e[1].elapsed_time(e[2]) for e in ev]
    cp = [e[2].elapsed_time(e[3]) for e in ev]
    step = [e[0].elapsed_time(e[1]) for e in whole]
    # a third pass splits the LM-head call at its phase marks: set-up kernels, the first GEMM
    # (the algorithmic pass), the acceptance kernels, the draw GEMM (T > 0), the last kernel
    ph = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    for e in ph:                      # torch creates the CUDA event on its first record
        for x in e:
            x.record()
    torch.cuda.synchronize()
    for i in range(steps):
        flush()
        e = ph[i]
        dev.attn()
        e[0].record()
        dev.lmhead_marked(e[1:5])
        e[5].record()
    torch.cuda.synchronize()
    names = ["setup", "gemm", "accept", "draw_gemm", "draw_pick"]
    phases = {n: [e[k].elapsed_time(e[k + 1]) for e in ph] for k, n in enumerate(names)}
    return dict(attn_ms=attn, lmhead_ms=lm, compact_ms=cp, step_ms=step, lmhead_phases=phases)


def time_e2e(dev, wl, steps, warmup, flush):
    """Same step through the C ABI with inputs in pinned host memory: the H2D copies of the step's
    inputs and the D2H copy of the accept results inside the timed region.  The step's inputs sit
    back to back in one device buffer, the attention's first: they go in one copy ahead of the
    attention call, and the LM head's inputs (hidden states, draft probabilities) in a second copy
    on a side stream that starts when the first ends and runs during the attention; the LM-head
    call waits for it.  The accept
    results come back in one copy."""
    host_in = torch.empty(dev.inputs.buf.shape, dtype=torch.uint8).pin_memory()
    host_in.copy_(dev.inputs.buf)
    host_out = torch.empty(dev.outputs.buf.shape, dtype=torch.uint8).pin_memory()
    h2d = host_in.numel()
    d2h = host_out.numel()
    cut = dev.inputs.offset("hidden")
    side = torch.cuda.Stream()
    main = torch.cuda.current_stream()

    def one():
        dev.inputs.buf[:cut].copy_(host_in[:cut], non_blocking=True)
        first = torch.cuda.Event()
        first.record(main)
        with torch.cuda.stream(side):
            # after the first copy (the two would share the link and delay the attention) and
            # after everything before it on the main stream (the previous step's reads)
            side.wait_event(first)
            dev.inputs.buf[cut:].copy_(host_in[cut:], non_blocking=True)
            ready = torch.cuda.Event()
            ready.record(side)
        dev.attn()
        main.wait_event(ready)
        dev.lmhead()
        dev.compact()
        host_out.copy_(dev.outputs.buf, non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        one()
        b.record()
        b.synchronize()
        ms.append(a.elapsed_time(b))
    return ms, h2d, d2h


def compact_layers_call(dev, wl, layers=64):
    """KV compaction over `layers` stacked layers with the step's real accept lengths and paths,
    into a compaction-only pool (every request given 64 free slots): returns the call."""
    from draft_tree_verification_masked_b200 import etree_kv_compact, make_batch
    B, hkv, D = wl.B, wl.hkv, wl.head_dim
    i32 = dict(dtype=torch.int32, device="cuda")
    kv0 = torch.zeros(B, **i32)
    cap = torch.full((B,), 64, **i32)
    sbase = torch.arange(B, dtype=torch.int64, device="cuda") * 64
    batch = make_batch(dev.cu_nodes, dev.parent, dev.tokens, kv0, sbase, cap, wl.n_max, 0)
    kt = torch.empty(layers, wl.n_total, hkv, D, dtype=torch.bfloat16, device="cuda")
    vt = torch.empty_like(kt)
    kt.normal_()
    vt.normal_()
    kc = torch.zeros(layers, B * 64, hkv, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    out = torch.empty(B, **i32)

    def one():
        etree_kv_compact(batch, dev.accept_len, dev.path, kt, vt, kc, vc, layers,
                         kt[0].numel(), kc[0].numel(), out, dev.ws)

    return one


def time_compact_layers(dev, wl, flush, layers=64, reps=10):
    """KV compaction over `layers` stacked layers (compact_layers_call), timed alone."""
    one = compact_layers_call(dev, wl, layers)
    for _ in range(3):
        one()
    torch.cuda.synchronize()
    tot = 0.0
    for _ in range(reps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        one()
        b.record()
        b.synchronize()
        tot += a.elapsed_time(b)
    us = tot / reps * 1e3
    acc = dev.accept_len.cpu().numpy()
    nbytes = compact_work(wl, acc, layers)
    del one
    torch.cuda.empty_cache()
    return us, nbytes


# -------------------------------------------------------------------------------- CPU oracle
def oracle_step(wl, requests, nthreads=0):
    """One oracle verification step over the listed requests: attention of all their rows,
    LM head + acceptance, compaction.  Returns accepted tokens (sum of a + 1)."""
    import oracle
    rows = []
    for r in requests:
        for g in range(int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])):
            for h in range(wl.hq):
                rows.append((g, h))
    rows = np.asarray(rows, dtype=np.int32)
    oracle.attention(wl.cu_nodes, wl.parent, wl.kv_len, wl.slot_base, wl.q, wl.k_tree,
                     wl.v_tree, wl.k_cache, wl.v_cache, wl.hq, wl.hkv,
                     oracle.scale_of(wl.head_dim), rows=rows, nthreads=nthreads)
    res = oracle.lmhead_accept(wl, requests, nthreads=nthreads)
    toks = 0
    for r in requests:
        o = res[r]
        a = int(o["accept_len"])
        toks += a + 1
        base, cap = int(wl.slot_base[r]), int(wl.slot_cap[r])
        a0, a1 = int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])
        sub_k = oracle._u16(wl.k_cache[base:base + cap]).copy()
        sub_v = oracle._u16(wl.v_cache[base:base + cap]).copy()
        oracle.kv_compact(np.array([0, a1 - a0], np.int32), wl.kv_len[r:r + 1],
                          np.zeros(1, np.int64), wl.slot_cap[r:r + 1], np.array([a], np.int32),
                          o["path"].reshape(1, 64), wl.k_tree[a0:a1], wl.v_tree[a0:a1], sub_k,
                          sub_v, 1, (a1 - a0) * wl.hkv * wl.head_dim,
                          cap * wl.hkv * wl.head_dim, wl.hkv, wl.head_dim)
    return toks


def sample_requests(wl, budget_rows=64):
    """A bounded sample: whole requests, in order, up to ~budget_rows tree nodes."""
    reqs, rows = [], 0
    for r in range(wl.B):
        if reqs and rows + wl.nodes(r) > budget_rows:
            break
        reqs.append(r)
        rows += wl.nodes(r)
    return reqs


def cpu_baseline(wl, min_seconds=10.0, max_reps=5):
    """The oracle on the host cores: one (`value_1core`, a single step of the sample), then all
    of them (`value`)."""
    import oracle
    reqs = sample_requests(wl)
    cores = oracle.max_threads()
    t1 = time.perf_counter()
    toks1 = oracle_step(wl, reqs, nthreads=1)
    dt1 = time.perf_counter() - t1
    # an explicit count: the one-core pass left the oracle's thread count at 1
    t0 = time.perf_counter()
    toks, reps = 0, 0
    while reps < max_reps and (reps == 0 or time.perf_counter() - t0 < min_seconds):
        toks += oracle_step(wl, reqs, nthreads=cores)
        reps += 1
    dt = time.perf_counter() - t0
    return {"value": toks / dt, "unit": "accepted tok/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{len(reqs)} of {wl.B} requests ({sum(wl.nodes(r) for r in reqs)} tree "
                      f"nodes) of workload {wl.name}, {reps} full oracle steps (attention all "
                      f"rows, LM head + acceptance, compaction), {dt:.1f} s",
            "value_1core": toks1 / dt1, "sample_1core": f"one step of the same sample, {dt1:.1f} s"}


# -------------------------------------------------------------------------------------- main
L2_POLICY = ("flushed before every timed step: 512 MiB write, then 256 MiB read (dirty lines "
             "written back before the timed region)")


def workload_config(name, wl, world):
    """The workload keys both arms' JSON lines carry in `config` (identical for both arms)."""
    return {"workload": name, "B": wl.B, "tree_nodes": int(wl.n_max),
            "kv_len": int(wl.kv_len_max), "hidden": wl.hidden_dim, "vocab": wl.vocab,
            "heads": f"{wl.hq}/{wl.hkv}", "head_dim": wl.head_dim,
            "temperature": wl.temperature, "layers": 1,
            "parallelism": f"dp{world} (independent requests per rank)", "l2": L2_POLICY}


def near_tie_rows(dev, wl):
    """T = 0: node rows whose top-1 / top-2 logit gap (the library's own node_gap) is below the
    near-tie bound 1e-3, where fp32 and fp64 may legitimately pick different argmaxes."""
    if wl.temperature != 0.0:
        return None
    gap = dev.node_gap.cpu().numpy()
    return {"rows": int(gap.size), "gap_lt_1e-3": int((gap < 1e-3).sum()),
            "min_gap": float(gap.min()) if gap.size else None}


def run_config(name, steps, warmup, peaks, rank, flush, with_e2e=True):
    from draft_tree_verification_masked_b200 import etree_attn_plan
    from draft_tree_verification_masked_b200 import workload as W
    from draft_tree_verification_masked_b200.runner import DeviceStep

    base, _, pg = name.partition("@p")                 # "<workload>@p<page size>": paged cache
    wl = W.generate(base, seed=W.config_seed(base) + 7919 * rank)
    # T > 0: every row's logits are kept (n_total x vocab fp32), so the bonus draw reads the stop
    # rows instead of a second pass over the head
    dev = DeviceStep(wl, page_size=int(pg) if pg else None, materialize=True)
    dev.step()
    st, det = dev.status()
    if st != 0:
        raise RuntimeError(f"device status {st} detail {det}")
    acc = dev.accept_len.cpu().numpy()
    toks = int((acc + 1).sum())
    t = time_steps(dev, steps, warmup, flush)
    plan = etree_attn_plan(dev.batch, wl.hq, wl.hkv)
    # attention + LM head (T=0: GEMM, fused accept; T>0 with every row materialised: prep, child
    # logits, GEMM, row merge, walk, draw over the stored rows) + compaction
    launches = plan["launches"] + (2 if wl.temperature == 0.0 else 6) + 1
    res = dict(wl=wl, dev=dev, toks=toks, t=t, plan=plan, launches=launches)
    if with_e2e:
        res["e2e"] = time_e2e(dev, wl, steps, max(3, warmup), flush)
    return res


def lowrank_report(name, flush, peaks, reps=20, warmup=3):
    """Device time of one etree_lowrank_candidates call (screen + exact rescoring of the k
    candidates) against its algorithmic bytes: |U| + |D| + |hidden| + the M k rows of W read."""
    from draft_tree_verification_masked_b200 import (etree_lowrank_candidates,
                                                     etree_lowrank_workspace_size,
                                                     etree_workspace_init)
    from draft_tree_verification_masked_b200 import workload as W
    lw = W.lowrank(name)
    dev = torch.device("cuda")
    h, D, U, Wt = (x.to(dev) for x in (lw.hidden, lw.D, lw.U, lw.W))
    ws = torch.zeros(etree_lowrank_workspace_size(lw.M, lw.H, lw.r, lw.V), dtype=torch.uint8,
                     device=dev)
    etree_workspace_init(ws)
    ids = torch.empty(lw.M, lw.k, dtype=torch.int32, device=dev)
    lg = torch.empty(lw.M, lw.k, dtype=torch.float32, device=dev)

    def one():
        etree_lowrank_candidates(h, D, U, Wt, lw.k, ids, lg, ws)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        one()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b) * 1e-3)
    t = statistics.mean(ts)
    nbytes = 2 * (lw.V * lw.r + lw.r * lw.H + lw.M * lw.H + lw.M * lw.k * lw.H)
    hbm = float(peaks["hbm_gbs"])
    return {"M": lw.M, "rank": lw.r, "k": lw.k, "vocab": lw.V, "hidden": lw.H,
            "us": t * 1e6, "bytes": nbytes, "GB/s": nbytes / t / 1e9,
            "hbm_frac": nbytes / t / 1e9 / hbm,
            "full_head_bytes": 2 * lw.V * lw.H}


def compact_layers_report(dev, wl, flush, peaks, layers=64):
    us, nbytes = time_compact_layers(dev, wl, flush, layers)
    hbm = float(peaks["hbm_gbs"])
    return {"layers": layers, "us": us, "GB/s": nbytes / us / 1e3, "hbm_frac": nbytes / us / 1e3 / hbm,
            "bytes": nbytes}


# Nominal B200 figures (HBM3e 7.7 TB/s, dense bf16 2.25 PFLOP/s), reported beside the measured
# ones for context; the roofline object uses the measured peaks.
NOMINAL_HBM_GBS = 7700.0
NOMINAL_BF16_TFLOPS = 2250.0


def kernel_report(wl, t, acc, peaks):
    hbm = float(peaks["hbm_gbs"])
    tc = float(peaks["bf16_tflops"])
    ab, af = attn_work(wl)
    lb, lf = lmhead_work(wl)
    cb = compact_work(wl, acc)
    am = statistics.mean(t["attn_ms"]) * 1e-3
    lm = statistics.mean(t["lmhead_ms"]) * 1e-3
    cm = statistics.mean(t["compact_ms"]) * 1e-3
    rep = {
        "attn": {"us": am * 1e6, "GB/s": ab / am / 1e9, "TFLOP/s": af / am / 1e12,
                 "hbm_frac": ab / am / 1e9 / hbm, "tc_frac": af / am / 1e12 / tc,
                 "bytes": ab, "flops": af},
        "lmhead": {"us": lm * 1e6, "GB/s": lb / lm / 1e9, "TFLOP/s": lf / lm / 1e12,
                   "hbm_frac": lb / lm / 1e9 / hbm, "tc_frac": lf / lm / 1e12 / tc,
                   "bytes": lb, "flops": lf},
        "compact": {"us": cm * 1e6, "GB/s": cb / cm / 1e9, "hbm_frac": cb / cm / 1e9 / hbm,
                    "bytes": cb},
    }
    # the LM-head call by phase (events between its kernels): the first GEMM against the
    # algorithmic work; the draw GEMM (T > 0) is implementation overhead, reported on its own
    # with the FLOPs it performs (2 B V H)
    ph = {n: statistics.mean(v) * 1e-3 for n, v in t["lmhead_phases"].items()}
    g1 = ph["gemm"]
    rep["lmhead_phases_us"] = {n: v * 1e6 for n, v in ph.items()}
    rep["lmhead_gemm"] = {"us": g1 * 1e6, "GB/s": lb / g1 / 1e9, "TFLOP/s": lf / g1 / 1e12,
                          "hbm_frac": lb / g1 / 1e9 / hbm, "tc_frac": lf / g1 / 1e12 / tc}
    if wl.temperature > 0.0:
        # the bonus draw reads each stop row's stored logits and its draft row (fp32)
        d = ph["draw_gemm"] + ph["draw_pick"]
        db = 8.0 * wl.B * wl.vocab
        rep["lmhead_draw"] = {"us": d * 1e6, "bytes": db, "GB/s": db / d / 1e9,
                              "hbm_frac": db / d / 1e9 / hbm,
                              "note": "bonus draw over the B stop rows' stored logits and draft "
                                      "rows; implementation overhead, not algorithmic"}
    for k in rep.values():
        if "GB/s" in k:
            k["hbm_frac_nominal"] = k["GB/s"] / NOMINAL_HBM_GBS
        if "TFLOP/s" in k:
            k["tc_frac_nominal"] = k["TFLOP/s"] / NOMINAL_BF16_TFLOPS
    return rep


def roofline(wl, rep, peaks, peak_kind, workload):
    dom = max(("attn", "lmhead", "compact"), key=lambda k: rep[k]["us"])
    k = rep[dom]
    hbm, tc = float(peaks["hbm_gbs"]), float(peaks["bf16_tflops"])
    traffic = ncu_traffic(dom, workload, kernel_source_hash(dom))
    if dom == "compact" or k["bytes"] / (hbm * 1e9) >= k.get("flops", 0) / (tc * 1e12):
        return {"kernel": dom, "bound": "hbm", "achieved": k["GB/s"], "peak": hbm,
                "unit": "GB/s", "frac": k["GB/s"] / hbm, "traffic": traffic,
                "algorithmic_bytes": k["bytes"], "peak_source": peak_kind}
    return {"kernel": dom, "bound": "tensor", "achieved": k["TFLOP/s"], "peak": tc,
            "unit": "TFLOP/s", "frac": k["TFLOP/s"] / tc, "traffic": traffic,
            "algorithmic_flops": k["flops"], "peak_source": peak_kind}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="etree", choices=["etree", "reference"])
    ap.add_argument("--config", default="dense27b_b1")
    ap.add_argument("--by-batch", default="batch64,conc512,tree64_t1,long32k,long128k,batch64@p16",
                    help="extra workloads measured in the same run (comma list, '' for none; "
                         "<workload>@p<N> runs it on a paged cache of N-token pages)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--lowrank", default="lowrank_r512,lowrank_r128",
                    help="low-rank candidate-head workloads timed after the step ('' for none)")
    ap.add_argument("--ncu-case", default="", choices=["", "attn", "lmhead", "compact64"],
                    help="profiling driver: run one step of --config, then only this call "
                         "--steps times (no flush, no timing, no JSON), for ncu captures")
    ap.add_argument("--ncu-kv", default="",
                    help="with --ncu-case: LO:HI replaces the workload's KV-length range (a "
                         "smaller capture of the same kernels)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.ncu_case:
        return ncu_case(args)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return main_reference(args, rank, world)

    import torch.distributed as dist
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    peaks, peak_kind = load_peaks()
    flush = L2Flush()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    main_res = run_config(args.config, args.steps, args.warmup, peaks, rank, flush)
    clk = clocks.stop()
    barrier()
    wl, t = main_res["wl"], main_res["t"]
    step_s = sum(t["step_ms"]) * 1e-3
    tokens = main_res["toks"] * args.steps
    e2e_ms, h2d, d2h = main_res["e2e"]
    e2e_s = sum(e2e_ms) * 1e-3
    step_s, e2e_s, tokens_all = reduce_over_ranks(step_s, e2e_s, tokens, world, "cuda")
    acc = main_res["dev"].accept_len.cpu().numpy()
    near = near_tie_rows(main_res["dev"], wl)
    rep = kernel_report(wl, t, acc, peaks)
    rep["compact_64layers"] = compact_layers_report(main_res["dev"], wl, flush, peaks)
    rl = roofline(wl, rep, peaks, peak_kind, args.config)
    head_plan, head_launches = main_res["plan"], main_res["launches"]

    by_batch = {}
    for name in [x for x in args.by_batch.split(",") if x]:
        del main_res["dev"]
        torch.cuda.empty_cache()
        # at most 10 steps per pass: the dense GEMM workloads are power-limited, and longer
        # sustained runs (25 steps per pass measured) read their second pass 5-15% slower
        r = run_config(name, max(3, min(10, args.steps)), max(3, min(5, args.warmup)), peaks,
                       rank, flush, with_e2e=False)
        racc = r["dev"].accept_len.cpu().numpy()
        rrep = kernel_report(r["wl"], r["t"], racc, peaks)
        rrep["compact_64layers"] = compact_layers_report(r["dev"], r["wl"], flush, peaks)
        sms = statistics.mean(r["t"]["step_ms"])
        by_batch[name] = {
            "B": r["wl"].B, "us_per_step": sms * 1e3,
            "us_per_step_median": statistics.median(r["t"]["step_ms"]) * 1e3,
            "accepted_tok_per_s": r["toks"] / (sms * 1e-3),
            "kernels": {k: {kk: round(vv, 4) if isinstance(vv, float) else vv
                            for kk, vv in v.items()} for k, v in rrep.items()},
            "roofline": roofline(r["wl"], rrep, peaks, peak_kind, name),
            "attn_plan": r["plan"], "gpu_launches_per_step": r["launches"],
            "near_ties": near_tie_rows(r["dev"], r["wl"]),
        }
        main_res = r

    lowrank = {}
    if args.lowrank:
        del main_res["dev"]
        torch.cuda.empty_cache()
        for name in [x for x in args.lowrank.split(",") if x]:
            lowrank[name] = lowrank_report(name, flush, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC,
        "value": tokens_all / step_s,
        "unit": "accepted tok/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_s / args.steps * 1e3,
        "us_per_step": step_s / args.steps * 1e6,
        "us_per_step_median": statistics.median(t["step_ms"]) * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; random-init LM head, N(0,1) activations and KV)",
        "config": workload_config(args.config, wl, world),
        "attn_plan": head_plan,
        "near_ties": near,
        "clocks": clk,
        "e2e": {"value": tokens_all / e2e_s, "unit": "accepted tok/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "us_per_step": e2e_s / args.steps * 1e6},
        "gpu_launches": head_launches * args.steps,
        "roofline": rl,
        "kernels": {k: {kk: round(vv, 4) if isinstance(vv, float) else vv for kk, vv in v.items()}
                    for k, v in rep.items()},
        "cpu_baseline": cpu,
        "by_batch": by_batch,
        "lowrank_head": lowrank,
    }
    print(json.dumps(line))


def ncu_case(args):
    """Runs one verification step of the workload, then the selected call alone `steps` times:
    the launches an ncu capture filters with -k / -s / -c.  compact64 moves the accepted rows of
    64 stacked layers."""
    from draft_tree_verification_masked_b200 import workload as W
    from draft_tree_verification_masked_b200.runner import DeviceStep
    base, _, pg = args.config.partition("@p")
    over = {}
    if args.ncu_kv:
        lo, hi = (int(x) for x in args.ncu_kv.split(":"))
        over["kv_len"] = (lo, hi)
    wl = W.generate(base, **over)
    dev = DeviceStep(wl, page_size=int(pg) if pg else None, materialize=True)   # as timed
    dev.step()
    st = dev.status()
    if st[0] != 0:
        raise RuntimeError(f"device status {st}")
    if args.ncu_case == "compact64":
        call = compact_layers_call(dev, wl, 64)
    else:
        call = {"attn": dev.attn, "lmhead": dev.lmhead}[args.ncu_case]
    for _ in range(args.steps):
        call()
    torch.cuda.synchronize()
    print(f"ncu case {args.config} {args.ncu_case} kv {args.ncu_kv or 'as configured'}: "
          f"{args.steps} calls")


def main_reference(args, rank, world):
    """The oracle arm: the fp64 CPU oracle on the same workload (rank 0 only)."""
    if rank != 0:
        return
    import oracle
    from draft_tree_verification_masked_b200 import workload as W
    wl = W.generate(args.config)
    reqs = sample_requests(wl)
    for _ in range(min(args.warmup, 1)):
        oracle_step(wl, reqs)
    times, toks = [], 0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        toks += oracle_step(wl, reqs)
        times.append(time.perf_counter() - t0)
    dt = sum(times)
    value = toks / dt
    line = {
        "metric": METRIC, "impl": "reference", "value": value, "unit": "accepted tok/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.config, wl, world),
        "cpu_baseline": {"value": value, "unit": "accepted tok/s", "cores": oracle.max_threads(),
                         "kind": "oracle",
                         "sample": f"{len(reqs)} of {wl.B} requests per step, full oracle "
                                   f"step (attention, LM head + acceptance, compaction)"},
        "e2e": {"value": value, "unit": "accepted tok/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


if __name__ == "__main__":
    main()
