"""Tree-sizing definitions for the tests -- TEST INFRASTRUCTURE ONLY (like the rest of oracle/).

The plain definition of the hardware-aware tree plan (a draft tree sized from measured draft and
verification costs: "EAGLE-4 官方推理代码发布 ...", arex-research.com, section
"投机树多大，由实测成本决定"), written independently of the library's planner:

* verification cost at (B, N, L): trilinear interpolation of the calibrated table, each axis
  extended linearly past its ends (the segment nearest to the point), clamped at 0;
* static tree of `depth` levels and `width` candidates per level: the rank-1 candidate continues
  the spine, ranks 2..width are leaves; at each level the target's token is the rank-k candidate
  with probability acc[k], independently;
* expected accepted drafts from the distribution of the stop level;
* the plan maximises B (E + 1) / (draft time + verification time), ties to fewer nodes, then
  fewer levels; depth 0 is plain decoding (one node, no draft time).
"""
from __future__ import annotations

import numpy as np


def _axis(grid, x):
    """Segment index and weights (w_lo, w_hi) of x on the grid; a one-point axis has (0, 1, 0)."""
    g = np.asarray(grid, dtype=np.float64)
    if len(g) == 1:
        return 0, 1.0, 0.0
    k = int(np.clip(np.searchsorted(g, x, side="left") - 1, 0, len(g) - 2))
    f = (x - g[k]) / (g[k + 1] - g[k])
    return k, 1.0 - f, f


def verify_cost(table, B, N, L):
    us = np.asarray(table["us"], dtype=np.float32).astype(np.float64)
    (ib, b0, b1), (in_, n0, n1), (il, l0, l1) = (_axis(table["B"], B), _axis(table["N"], N),
                                                 _axis(table["L"], L))
    tot = 0.0
    for db, wb in ((0, b0), (1, b1)):
        for dn, wn in ((0, n0), (1, n1)):
            for dl, wl in ((0, l0), (1, l1)):
                w = wb * wn * wl
                if w != 0.0:
                    tot += w * us[ib + db, in_ + dn, il + dl]
    return max(tot, 0.0)


def expected_accept(acc, depth, width):
    """E[accepted drafts] from the stop distribution: the walk reaches level j with probability
    s^(j-1) (s = acc[0]); there the spine continues (s), a side leaf ends the walk with j
    accepted (b = acc[1] + ... + acc[width-1]), or nothing matches and j - 1 are accepted."""
    acc = np.asarray(acc, dtype=np.float64)
    s = float(acc[0])
    b = float(acc[1:width].sum())
    e = 0.0
    for j in range(1, depth + 1):
        reach = s ** (j - 1)
        e += reach * (b * j + (1.0 - s - b) * (j - 1))
    return e + (s ** depth) * depth


def plan(table, B, L, acc, draft_us_per_level, draft_us_fixed=0.0, max_depth=16, max_width=16,
         max_nodes=64):
    best = None
    for d in range(0, max_depth + 1):
        for w in range(1, (1 if d == 0 else max_width) + 1):
            nodes = 1 + d * w
            if nodes > max_nodes:
                continue
            e = expected_accept(acc, d, w)
            step = (draft_us_fixed + d * draft_us_per_level if d else 0.0) + \
                verify_cost(table, B, nodes, L)
            tps = B * (e + 1.0) / step * 1e6 if step > 0 else 0.0   # no time: no rate
            if best is not None:
                bt = best["tokens_per_s"]
                better = tps > bt * (1 + 1e-12)
                tie = not better and tps >= bt * (1 - 1e-12)
                if not better and not (tie and (nodes, d) < (best["nodes"], best["depth"])):
                    continue
            best = dict(depth=d, width=w, nodes=nodes, expected_accept=e, step_us=step,
                        tokens_per_s=tps)
    return best
