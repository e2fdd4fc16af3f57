"""Pins for the fp64 oracle: checks against facts fixed outside the oracle itself.

Each check is chosen so that a plausible slip in the oracle (a dropped ancestor, the wrong parent
row, an inverted p/q ratio, a wrong Philox constant, an off-by-one in the compaction slots) fails
it.  Sources of truth: torch's fp64 scaled-dot-product attention with a mask built a different
way (positions, transitive closure), numpy's matmul, numpy's Philox4x64-10 bit generator, closed
forms of speculative sampling, chi-square tests and direct enumeration.  The pages (EAGLE-4
write-ups) print no worked example, so no stored values are used.
"""
import hashlib

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy import stats

import oracle
from draft_tree_verification_masked_b200 import workload as wlm

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


# --------------------------------------------------------------------------------------- Philox
def _minus_one(ctr):
    c = [int(x) for x in ctr]
    for i in range(4):
        if c[i] > 0:
            c[i] -= 1
            break
        c[i] = (1 << 64) - 1
    return np.array(c, dtype=np.uint64)


@pytest.mark.parametrize("ctr,key", [
    ([1, 0, 0, 0], [0, 0]),
    ([0, 0, 0, 0], [1, 2]),
    ([5, 7, 11, 1], [0xE7EE0004, 3]),
    ([2**64 - 1, 2**63, 12345, 2**40], [2**64 - 1, 2**64 - 1]),
])
def test_philox_matches_numpy_bit_generator(ctr, key):
    """numpy's Philox is Philox4x64-10; it advances the counter by one before each block."""
    ours = oracle.philox4x64(ctr, key)
    bg = np.random.Philox(counter=_minus_one(ctr), key=np.array(key, dtype=np.uint64))
    assert (bg.random_raw(4).astype(np.uint64) == ours).all()


def test_philox_random_counters_match_numpy():
    g = np.random.default_rng(7)
    for _ in range(200):
        ctr = g.integers(0, 2**63, size=4, dtype=np.uint64) + np.uint64(1)
        key = g.integers(0, 2**63, size=2, dtype=np.uint64)
        bg = np.random.Philox(counter=_minus_one(ctr), key=key)
        assert (bg.random_raw(4).astype(np.uint64) == oracle.philox4x64(ctr, key)).all()


def test_uniform_is_23bit_centred_exact_in_float32_and_uniform():
    us = np.array([oracle.uniform(0xE7EE0004, 9, r, r % 5, v, 0)
                   for r in range(400) for v in range(50)])
    assert (us > 0).all() and (us < 1).all()
    k = us * 2**23 - 0.5
    assert np.allclose(k, np.round(k), atol=0, rtol=0)
    # every value of the form (f + 1/2) 2^-23 survives a round trip through float32, and the
    # extreme fields stay strictly inside (0, 1)
    assert np.array_equal(us.astype(np.float32).astype(np.float64), us)
    top = np.float32((2**23 - 1 + 0.5) * 2.0**-23)
    assert float(top) == (2**23 - 0.5) * 2.0**-23 and top < 1.0
    counts, _ = np.histogram(us, bins=20, range=(0, 1))
    assert stats.chisquare(counts).pvalue > 1e-4
    # stream 1 and stream 0 are different draws
    assert oracle.uniform(1, 0, 0, 1, 0, 1) != oracle.uniform(1, 0, 0, 1, 0, 0)


# ------------------------------------------------------------------------------------- ancestry
def _closure(parent):
    n = len(parent)
    A = np.zeros((n, n), dtype=bool)
    for i in range(1, n):
        A[i, parent[i]] = True
    R = np.eye(n, dtype=bool)
    for _ in range(n):
        R = R | ((R.astype(np.int64) @ A.astype(np.int64)) > 0)
    return R


def test_ancestry_equals_transitive_closure():
    g = np.random.default_rng(3)
    for n, depth, branch, width in [(1, 0, None, None), (16, 6, 4, None), (64, 8, None, 16),
                                    (4, 3, 1, None), (64, 63, 1, None), (33, 5, 8, None)]:
        par = wlm.make_tree(n, depth, branch, width, g)
        st, anc, dep = oracle.ancestry(par)
        assert st == 0
        R = _closure(par)
        for i in range(n):
            bits = [(int(anc[i]) >> j) & 1 for j in range(n)]
            assert bits == list(R[i].astype(int)), (n, i)
            assert dep[i] == R[i].sum() - 1


@pytest.mark.parametrize("par", [[0, 0], [-1, 1], [-1, 0, 3, 1], [-1, -1], [-1, 0, 2]])
def test_ancestry_rejects_malformed(par):
    st, _, _ = oracle.ancestry(np.array(par, dtype=np.int32))
    assert st == oracle.EINVAL


# ------------------------------------------------------------------------------------ attention
def _small(n_nodes, depth, branch, B=2, hq=4, hkv=2, kv=(37, 37), seed=11, width=None):
    return wlm.generate("tiny", seed=seed, B=B, hq=hq, hkv=hkv, n_nodes=n_nodes, depth=depth,
                        depth_min=depth, branch=branch, width=width, kv_len=kv, hidden=64,
                        vocab=32)


def _f64(t):
    return t.to(torch.float64)


def _sdpa_rows(wl, r, mask_fn):
    """torch fp64 SDPA for every node/head of request r with the boolean mask from mask_fn."""
    a0, a1 = int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])
    n, L = a1 - a0, int(wl.kv_len[r])
    sb = int(wl.slot_base[r])
    G = wl.hq // wl.hkv
    outs = torch.zeros(n, wl.hq, wl.head_dim, dtype=torch.float64)
    lses = torch.zeros(n, wl.hq, dtype=torch.float64)
    mask = torch.as_tensor(mask_fn(n, L))
    for h in range(wl.hq):
        kvh = h // G
        K = torch.cat([_f64(wl.k_cache[sb:sb + L, kvh]), _f64(wl.k_tree[a0:a1, kvh])])
        Vv = torch.cat([_f64(wl.v_cache[sb:sb + L, kvh]), _f64(wl.v_tree[a0:a1, kvh])])
        Q = _f64(wl.q[a0:a1, h])
        scale = 1.0 / np.sqrt(wl.head_dim)
        o = F.scaled_dot_product_attention(Q[None, None], K[None, None], Vv[None, None],
                                           attn_mask=mask[None, None], scale=scale)
        outs[:, h] = o[0, 0]
        s = (Q @ K.T) * scale
        lses[:, h] = torch.logsumexp(s.masked_fill(~mask, float("-inf")), dim=1)
    return outs.numpy(), lses.numpy()


def _oracle_all(wl):
    out, lse, st = oracle.attention(wl.cu_nodes, wl.parent, wl.kv_len, wl.slot_base, wl.q,
                                    wl.k_tree, wl.v_tree, wl.k_cache, wl.v_cache, wl.hq, wl.hkv,
                                    oracle.scale_of(wl.head_dim))
    assert st == 0
    return out.reshape(-1, wl.hq, wl.head_dim), lse.reshape(-1, wl.hq)


def test_chain_tree_equals_causal_attention():
    """A chain is ordinary causal attention over [cache; chain] with positions compared."""
    wl = _small(n_nodes=6, depth=5, branch=1, kv=(37, 37))
    out, lse = _oracle_all(wl)

    def causal(n, L):
        qpos = L + np.arange(n)
        kpos = np.arange(L + n)
        return kpos[None, :] <= qpos[:, None]

    for r in range(wl.B):
        a0, a1 = int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])
        ref, ref_lse = _sdpa_rows(wl, r, causal)
        assert np.abs(out[a0:a1] - ref).max() < 1e-12
        assert np.abs(lse[a0:a1] - ref_lse).max() < 1e-12


def test_single_node_tree_equals_one_token_decode():
    wl = _small(n_nodes=1, depth=0, branch=None, kv=(50, 50), B=3)
    out, lse = _oracle_all(wl)
    for r in range(wl.B):
        ref, ref_lse = _sdpa_rows(wl, r, lambda n, L: np.ones((n, L + n), dtype=bool))
        assert np.abs(out[r:r + 1] - ref).max() < 1e-12
        assert np.abs(lse[r:r + 1] - ref_lse).max() < 1e-12


@pytest.mark.parametrize("n,depth,branch,width", [(16, 6, 4, None), (64, 8, None, 16),
                                                  (33, 4, 16, None)])
def test_tree_attention_equals_dense_closure_mask(n, depth, branch, width):
    wl = _small(n_nodes=n, depth=depth, branch=branch, width=width, kv=(20, 70), B=3, hq=6,
                hkv=2)
    out, lse = _oracle_all(wl)
    for r in range(wl.B):
        a0, a1 = int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])
        R = _closure(wl.parent[a0:a1])

        def closure_mask(n_, L):
            return np.concatenate([np.ones((n_, L), dtype=bool), R], axis=1)

        ref, ref_lse = _sdpa_rows(wl, r, closure_mask)
        assert np.abs(out[a0:a1] - ref).max() < 1e-12
        assert np.abs(lse[a0:a1] - ref_lse).max() < 1e-12


def test_attention_ignores_non_ancestors_and_sees_ancestors():
    wl = _small(n_nodes=16, depth=6, branch=4, B=1)
    out, _ = _oracle_all(wl)
    R = _closure(wl.parent)
    i = 15
    non = [j for j in range(16) if not R[i, j]]
    anc = [j for j in range(16) if R[i, j]]
    assert non and anc
    k2, v2 = wl.k_tree.clone(), wl.v_tree.clone()
    k2[non] = torch.randn(len(non), wl.hkv, wl.head_dim).to(torch.bfloat16)
    v2[non] = torch.randn(len(non), wl.hkv, wl.head_dim).to(torch.bfloat16)
    o2, _, _ = oracle.attention(wl.cu_nodes, wl.parent, wl.kv_len, wl.slot_base, wl.q, k2, v2,
                                wl.k_cache, wl.v_cache, wl.hq, wl.hkv, oracle.scale_of(128))
    o2 = o2.reshape(-1, wl.hq, 128)
    assert np.array_equal(o2[i], out[i])
    v3 = wl.v_tree.clone()
    v3[anc[-1]] += 1.0
    o3, _, _ = oracle.attention(wl.cu_nodes, wl.parent, wl.kv_len, wl.slot_base, wl.q, wl.k_tree,
                                v3, wl.k_cache, wl.v_cache, wl.hq, wl.hkv, oracle.scale_of(128))
    assert not np.array_equal(o3.reshape(-1, wl.hq, 128)[i], out[i])


def test_attention_row_subset_matches_full():
    wl = _small(n_nodes=16, depth=6, branch=4, B=2)
    out, lse = _oracle_all(wl)
    rows = np.array([[0, 0], [17, 3], [31, 1], [5, 2]], dtype=np.int32)
    o, l_, st = oracle.attention(wl.cu_nodes, wl.parent, wl.kv_len, wl.slot_base, wl.q,
                                 wl.k_tree, wl.v_tree, wl.k_cache, wl.v_cache, wl.hq, wl.hkv,
                                 oracle.scale_of(128), rows=rows)
    assert st == 0
    for k, (g, h) in enumerate(rows):
        assert np.array_equal(o[k], out[g, h]) and l_[k] == lse[g, h]


# -------------------------------------------------------------------------------------- LM head
def test_logits_equal_numpy_matmul():
    g = torch.Generator().manual_seed(5)
    hid = torch.randn(7, 300, generator=g).to(torch.bfloat16)
    w = (0.02 * torch.randn(1000, 300, generator=g)).to(torch.bfloat16)
    rows = np.array([6, 0, 3], dtype=np.int32)
    z = oracle.logits(hid, w, rows)
    ref = hid.double().numpy()[rows] @ w.double().numpy().T
    assert np.abs(z - ref).max() <= 1e-12 * np.abs(ref).max()


def test_row_top2_ties_and_order():
    z = np.array([[0.0, 1.0, 3.0, 3.0, -1.0], [5.0, 4.0, 4.0, 2.0, 5.0 - 1e-9]])
    arg, t1, t2 = oracle.row_top2(z)
    assert list(arg) == [2, 0]
    assert t1[0] == 3.0 and t2[0] == 3.0
    assert t1[1] == 5.0 and t2[1] == 5.0 - 1e-9


def _f_prefix(prefix, V):
    h = hashlib.sha256(np.array(prefix, dtype=np.int64).tobytes()).digest()
    return np.random.default_rng(int.from_bytes(h[:8], "little")).standard_normal(V)


@pytest.mark.parametrize("seed", range(12))
def test_greedy_walk_equals_sequential_greedy_decoding(seed):
    """Accepted tokens + bonus = what step-by-step greedy decoding emits (same logits)."""
    V = 16
    g = np.random.default_rng(100 + seed)
    n = int(g.integers(1, 40))
    while True:
        try:
            par = wlm.make_tree(n, int(g.integers(1, 10)), int(g.integers(1, 5)), None, g)
            break
        except ValueError:  # caps too tight for n nodes: draw again
            continue
    n = len(par)
    tok = np.zeros(n, dtype=np.int32)
    tok[0] = g.integers(V)
    prefix = {0: (int(tok[0]),)}
    for u in range(n):
        kids = [c for c in range(1, n) if par[c] == u]
        best = int(np.argmax(_f_prefix(prefix[u], V)))
        used = set()
        for c in kids:
            t = best if (best not in used and g.random() < 0.7) else None
            while t is None or t in used:
                t = int(g.integers(V))
            used.add(t)
            tok[c] = t
            prefix[c] = prefix[u] + (t,)
    z = np.stack([_f_prefix(prefix[i], V) for i in range(n)])
    arg, _, _ = oracle.row_top2(z)
    a, path, out = oracle.walk_greedy(par, tok, arg)
    # sequential greedy decoding from the root, no tree involved
    y, pre = [], (int(tok[0]),)
    for _ in range(n + 1):
        t = int(np.argmax(_f_prefix(pre, V)))
        y.append(t)
        pre = pre + (t,)
    # deepest tree node whose root path spells a prefix of y
    depth = {i: len(prefix[i]) - 1 for i in range(n)}
    consistent = [i for i in range(n) if list(prefix[i][1:]) == y[:depth[i]]]
    deepest = max(consistent, key=lambda i: depth[i])
    assert a == depth[deepest]
    assert list(out[:a + 1]) == y[:a + 1]
    assert path[a] == deepest and path[0] == 0
    assert (out[a + 1:] == -1).all() and (path[a + 1:] == -1).all()


def test_greedy_walk_duplicate_siblings_take_the_lowest_index():
    """Reading: when several children of the current node carry the argmax token, the walk takes
    the lowest node index.  Hand-worked tree: root 0 has children 1 (token 7), 2 (token 3) and
    3 (token 3); node 2 has child 4 (token 5), node 3 has child 5 (token 5).  The argmax rows are
    root -> 3, node 2 -> 5, node 3 -> 5, node 4 -> 9, node 5 -> 1, so the walk is 0 -> 2 -> 4
    and emits 3, 5 and the bonus 9 (through node 3 the bonus would be 1)."""
    par = np.array([-1, 0, 0, 0, 2, 3], dtype=np.int32)
    tok = np.array([0, 7, 3, 3, 5, 5], dtype=np.int32)
    arg = np.array([3, 0, 5, 5, 9, 1], dtype=np.int32)
    a, path, out = oracle.walk_greedy(par, tok, arg)
    assert a == 2 and list(path[:3]) == [0, 2, 4] and list(out[:3]) == [3, 5, 9]
    assert (path[3:] == -1).all() and (out[3:] == -1).all()


# ------------------------------------------------------------------------ stochastic acceptance
def _softmax(x):
    e = np.exp(x - x.max())
    return e / e.sum()


def _chain_trials(z_rows, q_rows, T, ntrial, seed, chunk=250_000):
    """Run ntrial requests of one chain (len = rows) with tokens drafted from q of the parent."""
    n, V = z_rows.shape
    g = np.random.default_rng(seed)
    firsts, seconds, alen = [], [], []
    done = 0
    step = 0
    while done < ntrial:
        m = min(chunk, ntrial - done)
        cu = (np.arange(m + 1) * n).astype(np.int32)
        par = np.tile(np.arange(-1, n - 1, dtype=np.int32), m)
        tok = np.zeros((m, n), dtype=np.int32)
        for k in range(1, n):
            c = np.cumsum(q_rows[k - 1].astype(np.float64))
            tok[:, k] = np.minimum(V - 1, np.searchsorted(c, g.random(m) * c[-1], side="right"))
        z = np.broadcast_to(z_rows, (m, n, V)).reshape(m * n, V)
        q = np.broadcast_to(q_rows, (m, n, V)).reshape(m * n, V)
        a, path, out, info = oracle.accept_chain_batch(cu, par, tok.reshape(-1), z, q, T,
                                                       seed, step)
        assert (a >= 0).all()
        firsts.append(out[:, 0])
        seconds.append(np.where(a >= 1, out[:, 1], -1))
        alen.append(a)
        done += m
        step += 1
    return np.concatenate(firsts), np.concatenate(seconds), np.concatenate(alen)


def _chisq_p(samples, probs):
    counts = np.bincount(samples, minlength=len(probs))
    exp = probs * len(samples)
    keep = exp > 0
    assert counts[~keep].sum() == 0
    return stats.chisquare(counts[keep], exp[keep]).pvalue


@pytest.mark.slow
@pytest.mark.parametrize("T", [1.0, 0.7])
def test_first_emitted_token_follows_target(T):
    """1e6 trials, V=16: the first emitted token ~ p_root, whatever the draft; the acceptance
    probability of the first draft equals sum_v min(p, q) (closed form)."""
    V = 16
    g = np.random.default_rng(21)
    z = g.normal(0, 1.5, size=(2, V))
    q = np.stack([_softmax(g.normal(0, 1.5, size=V)) for _ in range(2)]).astype(np.float32)
    first, _, a = _chain_trials(z, q, T, 1_000_000, seed=0xE7EE0100)
    p0 = _softmax(z[0] / T)
    assert _chisq_p(first, p0) > 1e-4
    acc = (a >= 1).mean()
    want = np.minimum(p0, q[0].astype(np.float64)).sum()
    assert abs(acc - want) < 5 * np.sqrt(want * (1 - want) / len(a))


@pytest.mark.slow
def test_second_emitted_token_follows_target_given_accepted_prefix():
    V = 16
    g = np.random.default_rng(22)
    T = 0.8
    z = g.normal(0, 1.5, size=(3, V))
    q = np.stack([_softmax(g.normal(0, 1.0, size=V)) for _ in range(3)]).astype(np.float32)
    first, second, a = _chain_trials(z, q, T, 1_000_000, seed=0xE7EE0200)
    assert _chisq_p(first, _softmax(z[0] / T)) > 1e-4
    sel = a >= 1
    assert _chisq_p(second[sel], _softmax(z[1] / T)) > 1e-4


@pytest.mark.slow
def test_identical_draft_is_always_accepted_and_bonus_follows_target():
    V = 16
    g = np.random.default_rng(23)
    z = g.normal(0, 1.0, size=(2, V))
    q = np.stack([_softmax(z[0]), _softmax(g.normal(size=V))]).astype(np.float32)
    # p uses fp64 softmax while q was rounded to fp32: both are the same distribution, so the
    # draft is accepted unless U*q >= p, which only rounding can cause.
    first, second, a = _chain_trials(z, q, 1.0, 400_000, seed=0xE7EE0300)
    assert (a >= 1).mean() > 0.9999
    sel = a == 1
    assert _chisq_p(second[sel], _softmax(z[1])) > 1e-4


@pytest.mark.slow
def test_exponential_race_is_an_exact_sampler():
    """10^6 races over 16 ids with zero weights: frequencies match w / sum w (exact
    multinomial)."""
    w = np.array([0.0, 1.0, 2.0, 0.0, 3.0, 0.5, 0.0, 4.0, 1e-3, 2.5, 0.0, 1.0, 0.25, 0.0, 6.0,
                  0.75])
    out = oracle.race_many(w, 1_000_000, 0xE7EE0400, 0, 0, 3)
    assert _chisq_p(out, w / w.sum()) > 1e-4
    assert oracle.race(np.zeros(16), 1, 0, 0, 0)[0] == -1


@pytest.mark.slow
@pytest.mark.parametrize("V", [300, 1000])
def test_exponential_race_is_an_exact_sampler_over_larger_vocabularies(V):
    """10^6 races: frequencies match w / sum w with zero weights and a zero run of 128 ids
    included; rare ids are pooled in groups of 16 for the test."""
    g = np.random.default_rng(V)
    w = g.exponential(size=V) * (g.random(V) < 0.8)
    w[128:256] = 0.0
    n = 1_000_000
    out = oracle.race_many(w, n, 0xE7EE0500, 0, 0, 2)
    probs = w / w.sum()
    if V <= 300:
        assert _chisq_p(out, probs) > 1e-4
    else:
        groups = np.arange(V) // 16
        assert _chisq_p(groups[out], np.bincount(groups, weights=probs)) > 1e-4
    assert (w[out] > 0).all()


def test_exponential_race_single_positive_weight_and_scale_invariance():
    """A single positive weight always wins; scaling every weight by the same factor keeps the
    winner (the race samples the normalised weights); the winner of w is never an id with
    w = 0."""
    g = np.random.default_rng(5)
    for trial in range(50):
        V = int(g.integers(2, 400))
        w = np.zeros(V)
        k = int(g.integers(V))
        w[k] = float(g.exponential())
        assert oracle.race(w, 7, trial, 3, 1)[0] == k
        w = g.exponential(size=V) * (g.random(V) < 0.5)
        if not (w > 0).any():
            continue
        t1 = oracle.race(w, 11, trial, 2, 0)[0]
        assert w[t1] > 0
        assert oracle.race(w * 1e-3, 11, trial, 2, 0)[0] == t1


def test_exponential_race_different_nodes_and_steps_draw_independently():
    """The race's uniforms are keyed by (seed, step) and counted by (id, node, request): over many
    requests the winners at two nodes (or two steps) agree only as often as independent draws
    would."""
    w = np.ones(64)
    n = 20_000
    a = oracle.race_many(w, n, 0xE7EE0600, 0, 0, 1)
    b = oracle.race_many(w, n, 0xE7EE0600, 0, 0, 2)
    c = oracle.race_many(w, n, 0xE7EE0600, 1, 0, 1)
    for x, y in ((a, b), (a, c)):
        same = (x == y).mean()
        assert abs(same - 1 / 64) < 5 * np.sqrt((1 / 64) * (63 / 64) / n), same


@pytest.mark.slow
def test_empty_residual_draws_the_bonus_from_the_target():
    """q = 2p (an over-confident draft that sums to 2): every residual max(0, p - q) is zero, so
    a rejected draft (U >= 1/2, probability 1/2) is answered by a draw from p itself; with the
    accepted drafts (x ~ q / 2 = p) the first emitted token follows p (chi-square, 2*10^5 trials),
    and after a rejection the bonus alone follows p too."""
    V = 16
    g = np.random.default_rng(24)
    z = g.normal(0, 1.5, size=(2, V))
    p0 = _softmax(z[0])
    q = np.stack([2 * p0, 2 * _softmax(z[1])]).astype(np.float32)
    n = 200_000
    cu = np.arange(0, 2 * n + 1, 2, dtype=np.int32)
    par = np.tile(np.array([-1, 0], dtype=np.int32), n)
    tok = np.zeros((n, 2), dtype=np.int32)
    tok[:, 1] = np.minimum(V - 1, np.searchsorted(np.cumsum(p0), g.random(n), side="right"))
    zz = np.broadcast_to(z, (n, 2, V)).reshape(2 * n, V)
    qq = np.broadcast_to(q, (n, 2, V)).reshape(2 * n, V)
    a, path, out, info = oracle.accept_chain_batch(cu, par, tok.reshape(-1), zz, qq, 1.0,
                                                   0xE7EE0700, 0)
    assert abs((a == 1).mean() - 0.5) < 5 * np.sqrt(0.25 / n)
    rej = a == 0
    assert (info[rej, 2] == 1).all()                   # every rejection fell back
    assert _chisq_p(out[rej, 0], p0) > 1e-4
    assert _chisq_p(out[:, 0], p0) > 1e-4
    # the tree rule takes the same fallback
    a2, path2, out2, info2, c2 = oracle.accept_tree_batch(cu, par, tok.reshape(-1), zz, qq, 1.0,
                                                          0xE7EE0700, 0)
    assert np.array_equal(a2, a) and np.array_equal(out2, out)


def test_accept_chain_rejects_branching_trees_and_bad_parents():
    z = np.zeros((3, 8))
    q = np.full((3, 8), 1 / 8, dtype=np.float32)
    tok = np.array([1, 2, 3], dtype=np.int32)
    a, *_ = oracle.accept_chain(np.array([-1, 0, 0], np.int32), tok, z, q, 1.0, 1, 0, 0)
    assert a == oracle.EUNSUPPORTED
    a, *_ = oracle.accept_chain(np.array([-1, 2, 1], np.int32), tok, z, q, 1.0, 1, 0, 0)
    assert a == oracle.EINVAL


def test_rejected_draft_residual_excludes_the_rejected_token_mass():
    """p = q except token 0 where the draft overshoots: a rejection can only bonus tokens with
    p > q, i.e. never token 0."""
    V = 8
    p = np.full(V, 1 / V)
    q = p.copy()
    q[0] += 0.3
    q[1:] -= 0.3 / (V - 1)
    z = np.log(np.stack([p, p]))
    tok = np.array([5, 0], dtype=np.int32)
    seen = set()
    for r in range(3000):
        a, path, out, info = oracle.accept_chain(np.array([-1, 0], np.int32), tok, z,
                                                 np.stack([q, q]).astype(np.float32), 1.0, 99, 0,
                                                 r)
        if a == 0:
            assert info[1] == 1 and out[0] != 0
            seen.add(int(out[0]))
    assert len(seen) == V - 1


# ------------------------------------------------------- stochastic acceptance on branching trees
def test_tree_rule_equals_chain_rule_on_chains():
    """On a chain the multi-candidate rule is the chain rule: same accepts, path, tokens, stop
    node, rejection flag and fallback, with c = 1 after the rejection (residual max(0, p - q))."""
    g = np.random.default_rng(31)
    for trial in range(300):
        n = int(g.integers(1, 9))
        V = int(g.integers(20, 300))
        T = float(g.choice([1.0, 0.7, 1.6]))
        z = g.normal(0, 2.0, size=(n, V))
        q = np.stack([_softmax(g.normal(0, 2.0, size=V)) for _ in range(n)]).astype(np.float32)
        par = np.arange(-1, n - 1, dtype=np.int32)
        tok = g.integers(0, V, size=n).astype(np.int32)
        for k in range(1, n):                     # draft most tokens from q so some are accepted
            if g.random() < 0.7:
                tok[k] = int(np.argmax(q[k - 1]))
        ac, pc, oc, ic = oracle.accept_chain(par, tok, z, q, T, 77, trial, 5)
        at, pt, ot, it, c = oracle.accept_tree(par, tok, z, q, T, 77, trial, 5)
        assert (ac, list(pc), list(oc)) == (at, list(pt), list(ot))
        assert list(ic) == list(it)
        assert c == (1.0 if ic[1] else 0.0)


def test_tree_rule_rejects_malformed_trees_and_tokens():
    z = np.zeros((3, 8))
    q = np.full((3, 8), 1 / 8, dtype=np.float32)
    a, *_ = oracle.accept_tree(np.array([-1, 2, 1], np.int32), np.array([1, 2, 3], np.int32), z,
                               q, 1.0, 1, 0, 0)
    assert a == oracle.EINVAL
    a, *_ = oracle.accept_tree(np.array([-1, 0, 0], np.int32), np.array([1, 2, 8], np.int32), z,
                               q, 1.0, 1, 0, 0)
    assert a == oracle.EINVAL


def _tree_trials(k, pz, qz, T, ntrial, seed, chunk=100_000):
    """ntrial requests of a two-level tree: the root has k children whose tokens are drafted
    independently from q_root; child with token x has 2 children drafted from q_x.  Target and
    draft logits depend on the token prefix only: root rows pz[0] / qz[0], rows after first token
    x pz[1 + x] / qz[1 + x].  Returns the first two emitted tokens and accept lengths."""
    V = pz.shape[1]
    g = np.random.default_rng(seed)
    q_of = np.stack([_softmax(r) for r in qz]).astype(np.float32)
    n = 1 + k + 2 * k
    par = np.array([-1] + [0] * k + [1 + i // 2 for i in range(2 * k)], dtype=np.int32)
    firsts, seconds, alen = [], [], []
    done, step = 0, 0
    while done < ntrial:
        m = min(chunk, ntrial - done)
        tok = np.zeros((m, n), dtype=np.int32)
        cq = np.cumsum(q_of.astype(np.float64), axis=1)
        tok[:, 1:1 + k] = np.minimum(V - 1, np.searchsorted(cq[0], g.random((m, k)) * cq[0, -1]))
        rowsel = np.zeros((m, n), dtype=np.int64)       # which prefix row each node uses
        for i in range(k):
            rowsel[:, 1 + i] = 1 + tok[:, 1 + i]
        for j in range(2 * k):
            parent_tok = tok[:, 1 + j // 2]
            u = g.random(m)
            t = np.empty(m, dtype=np.int64)
            for x in range(V):                          # inverse CDF of q_x, grouped by x
                sel = parent_tok == x
                t[sel] = np.searchsorted(cq[1 + x], u[sel] * cq[1 + x, -1])
            tok[:, 1 + k + j] = np.minimum(V - 1, t)
            rowsel[:, 1 + k + j] = 0                    # grandchildren are leaves: rows unused
        z = pz[rowsel.reshape(-1)]
        q = q_of[rowsel.reshape(-1)]
        cu = (np.arange(m + 1) * n).astype(np.int32)
        a, path, out, info, c = oracle.accept_tree_batch(cu, np.tile(par, m), tok.reshape(-1), z,
                                                          q, T, seed, step)
        assert (a >= 0).all()
        firsts.append(out[:, 0])
        seconds.append(np.where(a >= 1, out[:, 1], -1))
        alen.append(a)
        done += m
        step += 1
    return np.concatenate(firsts), np.concatenate(seconds), np.concatenate(alen)


@pytest.mark.slow
@pytest.mark.parametrize("k,T", [(2, 1.0), (3, 0.7), (4, 1.0)])
def test_multi_candidate_first_token_follows_target(k, T):
    """10^6 trials, V=16: with k candidates drafted independently from q_root (duplicates
    allowed), the first emitted token ~ p_root, through any number of sibling rejections and
    residual updates; given an accepted first token x, the second ~ p_x."""
    V = 16
    g = np.random.default_rng(40 + k)
    pz = g.normal(0, 1.5, size=(1 + V, V))
    qz = g.normal(0, 1.5, size=(1 + V, V))          # far from the target: many rejections
    first, second, a = _tree_trials(k, pz, qz, T, 1_000_000, seed=0xE7EE0600 + k)
    assert _chisq_p(first, _softmax(pz[0] / T)) > 1e-4
    acc = a >= 1
    assert 0.2 < acc.mean() < 0.99
    x = np.bincount(first[acc], minlength=V).argmax()
    sel = acc & (first == x)
    assert _chisq_p(second[sel], _softmax(pz[1 + x] / T)) > 1e-4


@pytest.mark.slow
def test_multi_candidate_sibling_acceptance_rates_match_the_closed_form():
    """10^6 trials of a root with two leaf children drafted independently from q, V=16.  The first
    child is accepted with probability A1 = sum min(p, q).  After its rejection the target is
    r1 = max(0, p - q) / (1 - A1) whatever token was rejected, and the second child, a fresh draw
    from q tested with a fresh uniform, is accepted with probability A2 = sum min(q, r1)."""
    V, T, m = 16, 1.0, 1_000_000
    g = np.random.default_rng(45)
    z = g.normal(0, 1.5, size=V)
    qv = _softmax(g.normal(0, 1.5, size=V)).astype(np.float32)
    p = _softmax(z / T)
    q64 = qv.astype(np.float64)
    A1 = np.minimum(p, q64).sum()
    r1 = np.maximum(0.0, p - q64) / (1.0 - A1)
    A2 = np.minimum(q64, r1).sum()
    cq = np.cumsum(q64)
    tok = np.zeros((m, 3), dtype=np.int32)
    tok[:, 1:] = np.minimum(V - 1, np.searchsorted(cq, g.random((m, 2)) * cq[-1]))
    cu = (np.arange(m + 1) * 3).astype(np.int32)
    par = np.tile(np.array([-1, 0, 0], dtype=np.int32), m)
    zz = np.broadcast_to(z, (3 * m, V))
    qq = np.broadcast_to(qv, (3 * m, V))
    a, path, out, info, c = oracle.accept_tree_batch(cu, par, tok.reshape(-1), zz, qq, T,
                                                      0xE7EE0700, 0)
    first = (path[:, 1] == 1).mean()
    second = (path[:, 1] == 2).mean()
    for got, want in ((first, A1), (second, (1 - A1) * A2)):
        assert abs(got - want) < 5 * np.sqrt(want * (1 - want) / m), (got, want)
    assert _chisq_p(out[:, 0], p) > 1e-4


def test_multi_candidate_identical_draft_accepts_the_first_child():
    """q = p at every node: the first child is always accepted (U q < p = q for U < 1)."""
    V = 32
    g = np.random.default_rng(50)
    z = g.normal(0, 1.0, size=(7, V))
    q = np.stack([_softmax(r) for r in z]).astype(np.float32)
    par = np.array([-1, 0, 0, 0, 1, 1, 2], dtype=np.int32)
    for r in range(500):
        tok = g.integers(0, V, size=7).astype(np.int32)
        a, path, out, info, c = oracle.accept_tree(par, tok, z, q, 1.0, 9, 0, r)
        assert path[1] == 1 and path[2] == 4 and a == 2 and info[1] == 0 and c == 0.0


def test_multi_candidate_residual_excludes_rejected_mass():
    """After the root's only candidate token is rejected by both siblings, the bonus comes from
    max(0, p - c q) with c = 1 + N(1) > 1: never token 0, where q exceeds p."""
    V = 8
    p = np.full(V, 1 / V)
    q = p.copy()
    q[0] += 0.3
    q[1:] -= 0.3 / (V - 1)
    z = np.log(np.stack([p, p, p]))
    qq = np.stack([q, q, q]).astype(np.float32)
    par = np.array([-1, 0, 0], dtype=np.int32)
    tok = np.array([5, 0, 0], dtype=np.int32)
    seen, two = set(), 0
    for r in range(4000):
        a, path, out, info, c = oracle.accept_tree(par, tok, z, qq, 1.0, 99, 0, r)
        if a == 0:
            assert out[0] != 0 and info[1] == 2 and c > 1.0
            seen.add(int(out[0]))
            two += 1
    assert two > 0 and len(seen) == V - 1


# ----------------------------------------------------------------------------------- compaction
def test_kv_compact_equals_numpy_gather():
    g = np.random.default_rng(9)
    B, hkv, d, layers = 5, 2, 8, 3
    n = np.array([1, 4, 16, 7, 64])
    cu = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    kv_len = g.integers(0, 40, size=B).astype(np.int32)
    cap = (kv_len + 64).astype(np.int32)
    base = np.concatenate([[0], np.cumsum(cap)[:-1]]).astype(np.int64)
    slots = int(base[-1] + cap[-1])
    a = np.array([0, 3, 5, 2, 63], dtype=np.int32)
    path = np.full((B, 64), -1, dtype=np.int32)
    for r in range(B):
        path[r, 0] = 0
        path[r, 1:a[r] + 1] = np.sort(g.choice(np.arange(1, n[r]), a[r], replace=False))
    tree_k = g.integers(0, 65535, size=(layers, cu[-1], hkv, d), dtype=np.uint16)
    tree_v = g.integers(0, 65535, size=(layers, cu[-1], hkv, d), dtype=np.uint16)
    ck = g.integers(0, 65535, size=(layers, slots, hkv, d), dtype=np.uint16)
    cv = g.integers(0, 65535, size=(layers, slots, hkv, d), dtype=np.uint16)
    ek, ev = ck.copy(), cv.copy()
    for r in range(B):
        dst = base[r] + kv_len[r] + np.arange(a[r] + 1)
        src = cu[r] + path[r, :a[r] + 1]
        ek[:, dst] = tree_k[:, src]
        ev[:, dst] = tree_v[:, src]
    st, newlen = oracle.kv_compact(cu, kv_len, base, cap, a, path, tree_k, tree_v, ck, cv, layers,
                                   cu[-1] * hkv * d, slots * hkv * d, hkv, d)
    assert st == 0
    assert np.array_equal(ck, ek) and np.array_equal(cv, ev)
    assert np.array_equal(newlen, kv_len + a + 1)


# ------------------------------------------------------------------------------ paged caches
def test_paged_attention_is_independent_of_page_placement():
    """The same logical caches scattered over shuffled pages of sizes 16 and 64 give bit-for-bit
    the contiguous attention (same keys, same order)."""
    wl = wlm.generate("tiny", B=4, n_nodes=[1, 6, 16, 9], depth=4, depth_min=2, branch=None,
                      width=8, kv_len=[0, 17, 100, 63], hidden=256, vocab=512)
    sc = oracle.scale_of(wl.head_dim)
    ref, lref, st = oracle.attention(wl.cu_nodes, wl.parent, wl.kv_len, wl.slot_base, wl.q,
                                     wl.k_tree, wl.v_tree, wl.k_cache, wl.v_cache, wl.hq, wl.hkv,
                                     sc)
    assert st == 0
    for P in (16, 64):
        pc = wlm.paged(wl, P, seed=P)
        out, lse, st = oracle.attention_paged(wl.cu_nodes, wl.parent, wl.kv_len, pc.block_table,
                                              P, wl.q, wl.k_tree, wl.v_tree, pc.k_pool,
                                              pc.v_pool, wl.hq, wl.hkv, sc)
        assert st == 0 and np.array_equal(out, ref) and np.array_equal(lse, lref)


def test_page_slots_by_hand():
    bt = np.array([[5, 2, 7], [0, 3, -1]], dtype=np.int32)
    assert list(oracle.page_slots(bt, 4, 0, [0, 3, 4, 9])) == [20, 23, 8, 29]
    assert list(oracle.page_slots(bt, 4, 1, [0, 5])) == [0, 13]


def test_paged_compaction_equals_contiguous_compaction_of_the_logical_cache():
    """Compacting into pages, then gathering each request's logical cache back through its block
    table, equals compacting the contiguous logical cache."""
    wl = wlm.generate("tiny", B=3, n_nodes=[5, 16, 2], depth=4, depth_min=2, branch=None,
                      width=8, kv_len=[14, 33, 0], hidden=256, vocab=512)
    P = 16
    pc = wlm.paged(wl, P, seed=1)
    a = np.array([2, 3, 1], dtype=np.int32)
    path = np.full((3, 64), -1, dtype=np.int32)
    path[0, :3] = [0, 1, 3]
    path[1, :4] = [0, 2, 5, 9]
    path[2, :2] = [0, 1]
    kt = oracle._u16(wl.k_tree)[None]
    vt = oracle._u16(wl.v_tree)[None]
    kpool = oracle._u16(pc.k_pool)[None].copy()
    vpool = oracle._u16(pc.v_pool)[None].copy()
    st, newlen = oracle.kv_compact_paged(wl.cu_nodes, wl.kv_len, pc.block_table, P, pc.slot_cap,
                                         a, path, kt, vt, kpool, vpool, 1)
    assert st == 0 and list(newlen) == list(wl.kv_len + a + 1)
    ck, cv = oracle._u16(wl.k_cache).copy(), oracle._u16(wl.v_cache).copy()
    d = wl.hkv * wl.head_dim
    st2, newlen2 = oracle.kv_compact(wl.cu_nodes, wl.kv_len, wl.slot_base, wl.slot_cap, a, path,
                                     wl.k_tree, wl.v_tree, ck, cv, 1, wl.n_total * d,
                                     ck.shape[0] * d, wl.hkv, wl.head_dim)
    assert st2 == 0 and list(newlen2) == list(newlen)
    for r in range(3):
        t = np.arange(int(newlen[r]))
        sl = oracle.page_slots(pc.block_table, P, r, t)
        b = int(wl.slot_base[r])
        assert np.array_equal(kpool[0, sl], ck[b + t]) and np.array_equal(vpool[0, sl], cv[b + t])


def test_kv_compact_capacity_overflow_leaves_request_untouched():
    cu = np.array([0, 4], dtype=np.int32)
    kv_len = np.array([10], dtype=np.int32)
    cap = np.array([12], dtype=np.int32)
    path = np.full((1, 64), -1, dtype=np.int32)
    path[0, :4] = [0, 1, 2, 3]
    tk = np.ones((4, 1, 8), dtype=np.uint16)
    ck = np.zeros((12, 1, 8), dtype=np.uint16)
    st, newlen = oracle.kv_compact(cu, kv_len, np.zeros(1, np.int64), cap, np.array([3], np.int32),
                                   path, tk, tk, ck, ck.copy(), 1, 32, 96, 1, 8)
    assert st == oracle.ENOSPACE and newlen[0] == 10 and not ck.any()


def test_kv_compact_fills_capacity_exactly_and_no_further():
    """kv_len + a + 1 == slot_cap is accepted; one slot short is refused and the request left
    untouched; no slot outside a request's written rows changes (the pool has spare slots past
    each capacity)."""
    cu = np.array([0, 4, 8], dtype=np.int32)
    kv_len = np.array([8, 8], dtype=np.int32)
    cap = np.array([12, 11], dtype=np.int32)
    base = np.array([0, 16], dtype=np.int64)
    a = np.array([3, 3], dtype=np.int32)
    path = np.full((2, 64), -1, dtype=np.int32)
    path[:, :4] = [0, 1, 2, 3]
    tk = (np.arange(8, dtype=np.uint16)[:, None, None] + 1) * np.ones((8, 1, 8), np.uint16)
    tv = tk + 100
    ck = np.zeros((32, 1, 8), dtype=np.uint16)
    cv = np.zeros((32, 1, 8), dtype=np.uint16)
    st, newlen = oracle.kv_compact(cu, kv_len, base, cap, a, path, tk, tv, ck, cv, 1, 64, 256,
                                   1, 8)
    assert st == oracle.ENOSPACE and list(newlen) == [12, 8]
    assert np.array_equal(ck[8:12], tk[0:4]) and np.array_equal(cv[8:12], tv[0:4])
    touched = np.zeros(32, dtype=bool)
    touched[8:12] = True
    assert not ck[~touched].any() and not cv[~touched].any()


# -------------------------------------------------------------------- low-rank candidate head
def _bf16_bits(x):
    return oracle._u16(torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16))


def _bits_value(b):
    return np.asarray(b, dtype=np.uint32).astype(np.uint32) << 16


def test_bf16_rounding_is_nearest_even():
    g = np.random.default_rng(61)
    xs = np.concatenate([g.normal(0, 3, 2000), g.normal(0, 1e-3, 500), [1.0 + 2 ** -8,
                         1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 2 ** -130, 3.5 * 2 ** -133]])
    for x in xs:
        b = oracle.bf16_round(float(x))
        v = np.frombuffer(np.uint32(b << 16).tobytes(), np.float32)[0]
        for nb in (b - 1, b + 1):                     # the bf16 neighbours (same sign)
            nv = np.frombuffer(np.uint32((nb & 0xFFFF) << 16).tobytes(), np.float32)[0]
            if np.isfinite(nv) and np.sign(nv) == np.sign(v):
                d, dn = abs(float(x) - float(v)), abs(float(x) - float(nv))
                assert d < dn or (d == dn and (b & 1) == 0), (x, v, nv)
    # fp32-exact inputs: the library's fp32 -> bf16 rounding agrees
    f = g.normal(0, 5, 5000).astype(np.float32)
    want = _bf16_bits(f)
    got = np.array([oracle.bf16_round(float(x)) for x in f], dtype=np.uint16)
    assert np.array_equal(got, want)


def test_lowrank_head_with_identity_factors_is_the_exact_top_k():
    """r = H, D = I and U = W: the screen is the exact logits, so the candidates are numpy's
    top-k of h W^T, in exact order."""
    g = np.random.default_rng(62)
    M, H, V, k = 5, 64, 300, 12
    hid = _bf16_bits(g.normal(size=(M, H)))
    W = _bf16_bits(g.normal(0, 0.3, size=(V, H)))
    D = _bf16_bits(np.eye(H))
    ids, lg, kth, _ = oracle.lowrank_candidates(hid, D, W, W, k)
    hf = hid.astype(np.uint32) << 16
    z = np.frombuffer(hf.tobytes(), np.float32).reshape(M, H).astype(np.float64) @ \
        np.frombuffer((W.astype(np.uint32) << 16).tobytes(), np.float32).reshape(V, H).astype(
            np.float64).T
    for m in range(M):
        order = np.lexsort((np.arange(V), -z[m]))[:k]
        assert list(ids[m]) == list(order)
        assert np.allclose(lg[m], z[m, order], rtol=0, atol=1e-9)


def test_lowrank_head_with_all_ids_is_the_exact_sort_and_permutes_with_the_vocab():
    g = np.random.default_rng(63)
    M, H, V, r = 3, 32, 48, 8
    hid = _bf16_bits(g.normal(size=(M, H)))
    D = _bf16_bits(g.normal(0, 0.2, size=(r, H)))
    U = _bf16_bits(g.normal(0, 0.2, size=(V, r)))
    W = _bf16_bits(g.normal(0, 0.2, size=(V, H)))
    ids, lg, _, _ = oracle.lowrank_candidates(hid, D, U, W, V)
    Wf = np.frombuffer((W.astype(np.uint32) << 16).tobytes(), np.float32).reshape(V, H)
    hf = np.frombuffer((hid.astype(np.uint32) << 16).tobytes(), np.float32).reshape(M, H)
    z = hf.astype(np.float64) @ Wf.astype(np.float64).T
    for m in range(M):
        assert list(ids[m]) == list(np.lexsort((np.arange(V), -z[m])))
    perm = g.permutation(V)
    ids2, lg2, _, _ = oracle.lowrank_candidates(hid, D, U[perm], W[perm], 10)
    ids1, lg1, _, _ = oracle.lowrank_candidates(hid, D, U, W, 10)
    assert np.array_equal(perm[ids2], ids1)          # the same tokens, renamed
    assert np.allclose(lg1, lg2, rtol=0, atol=1e-12)


def test_lowrank_screen_is_the_factorised_product():
    """U = I (r = V): the screen's logits are g = h D^T itself, unrounded.  Inputs are multiples
    of 1/8 in [-2, 2], so every product and sum is exact in fp64 and numpy's product is the
    definition; some of those values need more than bf16's 8 significant bits, so a screen that
    rounded g would differ.  D's rows repeat five distinct vectors, so each row's screen has
    groups of equal values and the top-k cut falls inside one: the screen keeps the lowest ids of
    that group.  The k survivors are then ordered by their exact logits h . W_c."""
    g = np.random.default_rng(64)
    M, H, V, k = 4, 64, 40, 6
    hv = g.integers(-16, 17, size=(M, H)) / 8.0
    dv = (g.integers(-16, 17, size=(5, H)) / 8.0)[g.integers(0, 5, size=V)]
    hid, D = _bf16_bits(hv), _bf16_bits(dv)
    U = _bf16_bits(np.eye(V))
    Wv = g.normal(0, 0.3, size=(V, H)).astype(np.float32)
    W = _bf16_bits(Wv)
    ids, lg, kth, za, gg = oracle.lowrank_candidates(hid, D, U, W, k, keep_approx=True,
                                                     keep_g=True)
    exact = hv @ dv.T
    rounded = torch.as_tensor(exact.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert not np.array_equal(rounded, exact)            # bf16 would change some values
    assert np.array_equal(za, exact) and np.array_equal(gg, exact)
    Wb = np.frombuffer((W.astype(np.uint32) << 16).tobytes(), np.float32).reshape(V, H)
    zx = hv @ Wb.astype(np.float64).T
    ties = 0
    for m in range(M):
        srt = np.lexsort((np.arange(V), -exact[m]))
        top = srt[:k]
        ties += int(exact[m, top[-1]] == exact[m, srt[k]])
        assert kth[m] == exact[m, top[-1]]
        assert sorted(ids[m]) == sorted(top)
        order = sorted(top, key=lambda c: (-zx[m, c], c))
        assert list(ids[m]) == order
        assert np.allclose(lg[m], zx[m, order], rtol=0, atol=1e-12)
    assert ties > 0                                      # the tie rule was exercised
