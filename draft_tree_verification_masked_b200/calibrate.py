"""Verification cost calibration: measured device time of one verification step over a grid of
batch sizes B, draft-tree sizes N (nodes per request, root included) and cached lengths L.

The draft tree's size should follow the measured cost of drafting and verifying at the running
batch size and hardware ("EAGLE-4 官方推理代码发布 ...", arex-research.com, section
"投机树多大，由实测成本决定": costs are measured online or by an offline calibration run once on
an idle GPU).  This module is that calibration for the verification side: it times
attention (one layer) + LM head with greedy acceptance + compaction (one layer) through the C ABI
on synthetic device-resident inputs and writes a JSON cost table that `etree_plan_tree` (and the
`plan_tree` binding) consume.

    python -m draft_tree_verification_masked_b200.calibrate --out table.json

Inputs are random (created on the device; timing does not depend on their values except through
acceptance, which only changes the compaction's few rows).  L2 is flushed before each timed step.
"""
from __future__ import annotations

import argparse
import json
import statistics
import time

import numpy as np
import torch

from . import (etree_kv_compact, etree_lmhead_accept, etree_verify_attn, etree_workspace_init,
               etree_workspace_size, make_batch)
from .workload import make_tree

DEFAULT_B = (1, 4, 16, 64, 256, 512)
DEFAULT_N = (1, 4, 8, 16, 32, 64)
DEFAULT_L = (1024, 4096, 16384)


class _Flush:
    def __init__(self):
        self.w = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
        self.r = torch.ones(64 << 20, dtype=torch.int32, device="cuda")
        self.s = torch.empty((), dtype=torch.int64, device="cuda")

    def __call__(self):
        self.w.zero_()
        torch.sum(self.r, dim=0, dtype=torch.int64, out=self.s)


def time_step(B, N, L, w_lm, hq, hkv, H, flush, reps=5, warmup=2, seed=0):
    """Median device µs of one verification step for B requests of N-node trees over L cached
    tokens each."""
    dev = torch.device("cuda")
    V = w_lm.shape[0]
    g = np.random.default_rng([seed, B, N, L])
    par = np.concatenate([make_tree(N, min(N - 1, 8), None, 16, g) for _ in range(B)])
    cu = np.arange(B + 1, dtype=np.int32) * N
    i32 = dict(dtype=torch.int32, device=dev)
    cu_t = torch.as_tensor(cu, **i32)
    par_t = torch.as_tensor(par.astype(np.int32), **i32)
    tok_t = torch.randint(0, V, (B * N,), **i32)
    kv_t = torch.full((B,), L, **i32)
    cap = L + N + 1
    base_t = torch.arange(B, dtype=torch.int64, device=dev) * cap
    cap_t = torch.full((B,), cap, **i32)
    batch = make_batch(cu_t, par_t, tok_t, kv_t, base_t, cap_t, N, L)
    bf = torch.bfloat16
    q = torch.randn(B * N, hq, 128, dtype=bf, device=dev)
    kt = torch.randn(B * N, hkv, 128, dtype=bf, device=dev)
    vt = torch.randn_like(kt)
    kc = torch.randn(B * cap, hkv, 128, dtype=bf, device=dev)
    vc = torch.randn_like(kc)
    hid = torch.randn(B * N, H, dtype=bf, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(B * N, hq, dtype=torch.float32, device=dev)
    acc = torch.empty(B, **i32)
    path = torch.empty(B, 64, **i32)
    otok = torch.empty(B, 65, **i32)
    klen = torch.empty(B, **i32)
    ws = torch.zeros(etree_workspace_size(batch, hq, hkv, 128, H, V), dtype=torch.uint8,
                     device=dev)
    etree_workspace_init(ws)
    scale = 128 ** -0.5

    def step():
        etree_verify_attn(batch, q, kt, vt, kc, vc, scale, out, lse, ws)
        etree_lmhead_accept(batch, hid, w_lm, 0.0, None, 1, 0, acc, path, otok, None, None, ws)
        etree_kv_compact(batch, acc, path, kt, vt, kc, vc, 1, kt.numel(), kc.numel(), klen, ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        step()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b) * 1e3)
    return statistics.median(ts)


def calibrate(Bs=DEFAULT_B, Ns=DEFAULT_N, Ls=DEFAULT_L, hq=40, hkv=8, H=5120, V=151936,
              reps=5, log=None):
    """Returns the cost table: {"B": [...], "N": [...], "L": [...], "us": [[[...]]] (B, N, L),
    "shape": {...}, "device": name}."""
    torch.cuda.init()
    w_lm = (torch.randn(V, H, dtype=torch.bfloat16, device="cuda") * 0.02)
    flush = _Flush()
    us = np.zeros((len(Bs), len(Ns), len(Ls)))
    for i, B in enumerate(Bs):
        for j, N in enumerate(Ns):
            for k, L in enumerate(Ls):
                t0 = time.time()
                us[i, j, k] = time_step(B, N, L, w_lm, hq, hkv, H, flush, reps=reps)
                torch.cuda.empty_cache()
                if log:
                    log(f"B={B} N={N} L={L}: {us[i, j, k]:.1f} us ({time.time() - t0:.1f} s)")
    return {"B": list(Bs), "N": list(Ns), "L": list(Ls), "us": us.round(2).tolist(),
            "shape": {"hq": hq, "hkv": hkv, "head_dim": 128, "hidden": H, "vocab": V},
            "step": "attention (1 layer) + LM head with greedy acceptance + compaction (1 layer)",
            "device": torch.cuda.get_device_name()}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--out", required=True)
    ap.add_argument("--B", default=",".join(map(str, DEFAULT_B)))
    ap.add_argument("--N", default=",".join(map(str, DEFAULT_N)))
    ap.add_argument("--L", default=",".join(map(str, DEFAULT_L)))
    ap.add_argument("--reps", type=int, default=5)
    args = ap.parse_args()
    ints = lambda s: tuple(int(x) for x in s.split(","))
    table = calibrate(ints(args.B), ints(args.N), ints(args.L), reps=args.reps,
                      log=lambda m: print(m, flush=True))
    with open(args.out, "w") as f:
        json.dump(table, f, indent=1)


if __name__ == "__main__":
    main()
