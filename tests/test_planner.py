"""Hardware-aware tree sizing (host only): the oracle's plain definition pinned by closed forms,
a Monte-Carlo walk and multilinear tables; the library's planner against it."""
import itertools

import numpy as np
import pytest

import draft_tree_verification_masked_b200 as et
from oracle import planner as OP


def _table(f, B=(1, 4, 16, 64), N=(1, 4, 16, 64), L=(512, 4096)):
    us = np.array([[[f(b, n, l) for l in L] for n in N] for b in B], dtype=np.float32)
    return {"B": list(B), "N": list(N), "L": list(L), "us": us.tolist()}


@pytest.mark.parametrize("s,b,d", [(1.0, 0.0, 5), (0.0, 0.3, 4), (0.6, 0.0, 7), (0.5, 0.2, 3)])
def test_expected_accept_closed_forms(s, b, d):
    acc = [s, b]
    e = OP.expected_accept(acc, d, 2)
    if s == 1.0:
        want = d
    elif s == 0.0:
        want = b                                     # only level 1 is tested
    else:                                            # sum_j s^(j-1) (s + b)
        want = (s + b) * (1 - s ** d) / (1 - s)
    assert abs(e - want) < 1e-12


def test_expected_accept_matches_a_simulated_walk():
    g = np.random.default_rng(7)
    acc = np.array([0.55, 0.15, 0.08, 0.05])
    for d, w in [(1, 1), (3, 2), (6, 4), (8, 1)]:
        n = 200_000
        ranks = g.choice(len(acc) + 1, size=(n, d), p=np.append(acc, 1 - acc.sum()))
        got = np.zeros(n)
        alive = np.ones(n, bool)
        for j in range(d):
            r = ranks[:, j]
            spine = alive & (r == 0)
            side = alive & (r >= 1) & (r < w)
            got += spine + side
            alive = spine
        sd = got.std() / np.sqrt(n)
        assert abs(got.mean() - OP.expected_accept(acc, d, w)) < 5 * sd + 1e-9


def test_interpolation_is_exact_on_multilinear_tables():
    f = lambda b, n, l: 100 + 3 * b + 5 * n + 0.01 * l + 0.02 * b * n + 1e-4 * n * l
    t = _table(f)
    for B, N, L in [(1, 1, 512), (7, 9, 1000), (64, 64, 4096), (100, 80, 9000), (2, 3, 100)]:
        assert abs(OP.verify_cost(t, B, N, L) - f(B, N, L)) < 1e-6 * f(B, N, L)
        assert abs(et.etree_verify_cost(t, B, N, L) - f(B, N, L)) < 1e-6 * f(B, N, L)


def test_plan_extremes():
    flat = _table(lambda b, n, l: 1000.0)
    # no acceptance: plain decoding
    p = OP.plan(flat, 8, 1024, [0.0], 50.0)
    assert (p["depth"], p["nodes"]) == (0, 1)
    # certain acceptance of the top draft, free drafting, flat verification: deepest chain
    p = OP.plan(flat, 8, 1024, [1.0], 0.0, max_depth=16, max_width=4)
    assert (p["depth"], p["width"]) == (16, 1) and p["expected_accept"] == 16
    # verification cost growing with nodes at large B narrows the tree
    steep = _table(lambda b, n, l: 200.0 + 0.5 * b * n)
    acc = [0.5, 0.15, 0.08, 0.05, 0.03, 0.02]
    small = OP.plan(steep, 1, 1024, acc, 30.0)
    large = OP.plan(steep, 64, 1024, acc, 30.0)
    assert small["nodes"] > large["nodes"]


def test_library_planner_equals_oracle_on_random_tables():
    g = np.random.default_rng(11)
    for trial in range(60):
        B = tuple(sorted(g.choice(np.arange(1, 600), size=g.integers(1, 5), replace=False)))
        N = tuple(sorted(g.choice(np.arange(1, 65), size=g.integers(1, 5), replace=False)))
        L = tuple(sorted(g.choice(np.arange(1, 20000), size=g.integers(1, 4), replace=False)))
        base = g.uniform(50, 500)
        t = _table(lambda b, n, l: base + g.uniform(0, 3) * b * n + g.uniform(0, 1e-2) * l
                   + g.uniform(0, 20) * n, B, N, L)
        k = int(g.integers(1, 8))
        acc = g.dirichlet(np.ones(k + 1))[:k] * g.uniform(0.3, 1.0)
        for Bq, Lq in [(int(g.integers(1, 700)), int(g.integers(0, 30000))) for _ in range(3)]:
            args = dict(draft_us_per_level=float(g.uniform(0, 300)),
                        draft_us_fixed=float(g.uniform(0, 100)),
                        max_depth=int(g.integers(0, 12)), max_width=int(g.integers(1, 16)),
                        max_nodes=int(g.integers(1, 65)))
            acc32 = np.asarray(acc, dtype=np.float32)
            o = OP.plan(t, Bq, Lq, acc32, **args)
            c = et.etree_plan_tree(t, Bq, Lq, acc32, **args)
            assert (c["depth"], c["width"], c["nodes"]) == (o["depth"], o["width"], o["nodes"])
            for key in ("expected_accept", "step_us", "tokens_per_s"):
                assert abs(c[key] - o[key]) <= 1e-6 * max(1.0, abs(o[key])), (key, c, o)


def test_packaged_b200_table_narrows_the_tree_as_the_batch_grows():
    t = et.load_cost_table("b200_dense27b")
    acc = [0.55, 0.12, 0.06, 0.04, 0.03, 0.02, 0.015, 0.01]
    plans = {B: et.etree_plan_tree(t, B, 4096, acc, 30.0, max_depth=12, max_width=8)
             for B in (1, 16, 64, 512)}
    assert plans[1]["nodes"] >= plans[64]["nodes"] >= plans[512]["nodes"]
    assert plans[1]["nodes"] > plans[512]["nodes"]


def test_planner_rejects_bad_arguments():
    t = _table(lambda b, n, l: 100.0)
    with pytest.raises(et.EtreeError):
        et.etree_plan_tree(t, 0, 100, [0.5], 10.0)
    with pytest.raises(et.EtreeError):
        et.etree_plan_tree(t, 4, 100, [0.7, 0.5], 10.0)          # mass above 1
    bad = dict(t, B=[4, 1, 16, 64])
    with pytest.raises(et.EtreeError):
        et.etree_verify_cost(bad, 4, 4, 100)
