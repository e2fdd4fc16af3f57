"""The seeded input generator against its stated recipe (no GPU): tree shapes and caps, the T=0
draft tokens and planted argmax, the T>0 draft sampling, the cache slot layout, page placement,
and determinism.  The generator holds none of the method's arithmetic; these checks only make
sure the inputs are what the workload descriptions say they are."""
import numpy as np
import pytest
import torch

from draft_tree_verification_masked_b200 import workload as W


def _depths(par):
    d = np.zeros(len(par), dtype=np.int64)
    for i in range(1, len(par)):
        d[i] = d[par[i]] + 1
    return d


@pytest.mark.parametrize("n,depth,branch,width", [(16, 6, 4, None), (64, 8, None, 16),
                                                  (4, 3, 1, None), (1, 0, None, None),
                                                  (33, 5, 8, None), (64, 63, 1, None)])
def test_trees_are_bfs_ordered_and_respect_their_caps(n, depth, branch, width):
    g = np.random.default_rng(n * 100 + depth)
    for _ in range(20):
        par = W.make_tree(n, depth, branch, width, g)
        assert len(par) == n and par[0] == -1
        assert all(0 <= par[i] < i for i in range(1, n))
        d = _depths(par)
        assert (np.diff(d) >= 0).all()                       # BFS: depth never decreases
        assert d.max() == min(depth, n - 1)                  # the spine reaches the depth cap
        kids = np.bincount(par[1:], minlength=n)
        if branch is not None:
            assert kids.max() <= branch
        if width is not None:
            assert np.bincount(d).max() <= width
        # BFS order: the children of earlier nodes come first
        assert list(par[1:]) == sorted(par[1:])


def test_tree_caps_that_leave_no_room_are_refused():
    with pytest.raises(ValueError):
        W.make_tree(10, 2, 1, None, np.random.default_rng(0))
    with pytest.raises(ValueError):
        W.make_tree(0, 2, None, None, np.random.default_rng(0))


def test_greedy_draft_tokens_match_the_recipe():
    """Siblings carry distinct tokens, at most one of them the parent's planted token, and the
    first child carries it with the configured match probability."""
    g = np.random.default_rng(5)
    V, m = 50, 0.7
    firsts, matches = 0, 0
    for trial in range(400):
        par = W.make_tree(16, 6, 4, None, g)
        planted = g.integers(V, size=16).astype(np.int32)
        tok = W._draft_tokens_greedy(par, planted, V, m, g)
        assert ((tok >= 0) & (tok < V)).all()
        for u in range(16):
            kids = [c for c in range(1, 16) if par[c] == u]
            if not kids:
                continue
            ts = [int(tok[c]) for c in kids]
            assert len(set(ts)) == len(ts)
            assert ts.count(int(planted[u])) <= 1
            firsts += 1
            matches += ts[0] == planted[u]
    rate = matches / firsts
    assert abs(rate - m) < 5 * np.sqrt(m * (1 - m) / firsts)


def test_planted_token_is_the_argmax_of_the_greedy_workloads():
    wl = W.generate("tiny", B=3, n_nodes=[16, 5, 1])
    z = wl.hidden.double().numpy() @ wl.w_lm.double().numpy().T
    assert (z.argmax(axis=1) == wl.planted).all()
    assert wl.q_draft is None and wl.temperature == 0.0


def test_stochastic_draft_tokens_are_drawn_from_the_parent_distribution():
    """For x ~ q, E[q(x)] = sum_v q(v)^2: the sample mean over many children matches it, and
    every drawn token has positive draft probability under its parent's row."""
    wl = W.generate("conc512", B=400, n_nodes=4, hidden=64, vocab=16, kv_len=(1, 4), hq=2,
                    hkv=1)
    q = wl.q_draft.double().numpy()
    got, want = [], []
    for r in range(wl.B):
        a, b = int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])
        for i in range(a + 1, b):
            row = q[a + int(wl.parent[i])]
            got.append(row[wl.tokens[i]])
            want.append((row ** 2).sum())
    got, want = np.array(got), np.array(want)
    assert (got > 0).all()
    assert abs(got.mean() - want.mean()) < 5 * got.std() / np.sqrt(len(got))
    assert np.allclose(q.sum(axis=1), 1.0, atol=1e-5)


def test_cache_slots_are_disjoint_and_sized_for_a_full_step():
    wl = W.generate("batch64", B=8, hidden=64, vocab=300)
    lo, hi = W.CONFIGS["batch64"]["kv_len"]
    assert ((wl.kv_len >= lo) & (wl.kv_len <= hi)).all()
    assert (wl.slot_cap == wl.kv_len + 64).all()             # room for root + 63 accepted
    ends = wl.slot_base + wl.slot_cap
    assert wl.slot_base[0] == 0 and (wl.slot_base[1:] == ends[:-1]).all()
    assert wl.slots == int(ends[-1])
    assert wl.n_total == int(wl.cu_nodes[-1]) == wl.q.shape[0] == wl.hidden.shape[0]


def test_generation_is_deterministic_and_independent_of_threads(monkeypatch):
    a = W.normal_f32(3_000_000, 0.5, 123, "q")
    monkeypatch.setattr(W, "_threads", lambda: 1)
    b = W.normal_f32(3_000_000, 0.5, 123, "q")
    assert np.array_equal(a, b)
    w1 = W.generate("tiny", B=2, n_nodes=[7, 3], hidden=64, vocab=256)
    w2 = W.generate("tiny", B=2, n_nodes=[7, 3], hidden=64, vocab=256)
    for f in ("parent", "tokens", "kv_len", "planted"):
        assert np.array_equal(getattr(w1, f), getattr(w2, f)), f
    for f in ("q", "k_cache", "hidden", "w_lm"):
        assert torch.equal(getattr(w1, f), getattr(w2, f)), f
    w3 = W.generate("tiny", seed=W.config_seed("tiny") + 1, B=2, n_nodes=[7, 3], hidden=64,
                    vocab=256)
    assert not torch.equal(w1.q, w3.q)


def test_bf16_tensors_are_nearest_even_roundings_of_fp32_normals():
    f = W.normal_f32(1000, 2.0, 77, "k_tree")
    b = W.normal_bf16((1000,), 2.0, 77, "k_tree")
    bits = W.bf16_bits(b).astype(np.uint32)
    u = f.view(np.uint32)
    # round to nearest even on the upper 16 bits of each fp32 value (no NaN or Inf here)
    want = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    assert np.array_equal(bits, want.astype(np.uint32))
    assert abs(f.std() - 2.0) < 0.2


@pytest.mark.parametrize("P", [16, 64])
def test_paged_layout_holds_each_request_cache_at_distinct_pages(P):
    wl = W.generate("tiny", B=4, n_nodes=[1, 6, 16, 9], depth=4, depth_min=2, branch=None,
                    width=8, kv_len=[0, 17, 100, 63], hidden=64, vocab=256)
    pc = W.paged(wl, P, seed=P)
    mapped = pc.block_table[pc.block_table >= 0]
    assert len(set(mapped.tolist())) == len(mapped)           # no page shared
    assert pc.num_pages == len(mapped) + 3                     # plus the unmapped spares
    assert (pc.slot_cap >= wl.slot_cap).all() and (pc.slot_cap % P == 0).all()
    for r in range(wl.B):
        base = int(wl.slot_base[r])
        for t in range(int(wl.slot_cap[r])):
            s = int(pc.block_table[r, t // P]) * P + t % P
            assert torch.equal(pc.k_pool[s], wl.k_cache[base + t])
            assert torch.equal(pc.v_pool[s], wl.v_cache[base + t])


def test_lowrank_factors_have_the_head_scale():
    lw = W.lowrank("lowrank_tiny", H=512, r=64, V=2048)
    ud = lw.U.double() @ lw.D.double()
    assert lw.hidden.shape == (lw.M, lw.H) and lw.D.shape == (lw.r, lw.H)
    assert lw.U.shape == (lw.V, lw.r) and lw.W.shape == (lw.V, lw.H)
    assert abs(float(ud.std()) - 0.02) < 0.002
    resid = lw.W.double() - ud
    assert 0.004 < float(resid.std()) < 0.006                  # W = U D + N(0, 0.005)
