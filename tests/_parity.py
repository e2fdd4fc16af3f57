"""Comparisons of the CUDA path against the fp64 oracle (test infrastructure).

Tolerances:
* attention output: max-abs <= 2e-2 and relative RMS <= 5e-3 against fp64 (bf16 inputs and
  output, fp32 accumulation); lse: |err| <= 1e-3 (fp32 softmax statistics over <= 131k keys);
* argmax, paths, accept lengths, bonus tokens, compacted KV: bit-exact, except at logit near-ties
  (fp64 top1 - top2 < 1e-3), which are logged and counted and excuse the rest of that request;
* per-node top1-top2 gap: |err| <= 1e-3 + 1e-3 |gap| (fp32 accumulation over hidden_dim);
* T > 0: accept decisions and drawn tokens bit-exact, except sampling near-ties where the fp64
  quantities compared differ by less than 1e-5 relative (fp32 vs fp64 rounding): U*q vs p for
  an accept test, or the two ids' exponential-race keys (plus the fp32 error of the weights).
"""
from __future__ import annotations

import numpy as np

import oracle

# Near-tie records of the session, printed by the terminal summary (tests/conftest.py).
NEAR_LOG: list[dict] = []

ATTN_MAX_ABS = 2e-2
ATTN_REL_RMS = 5e-3
LSE_ABS = 1e-3
NEAR_TIE = 1e-3
SAMPLE_REL = 1e-5


def log_near(label, wl, res, ores, requests, excused):
    """Records one comparison's near-tie counts: requests checked, decisions whose fp64 margin is
    under the near-tie bound (T = 0: nodes with top1 - top2 < NEAR_TIE; T > 0: not counted
    separately), and requests excused by a replayed near-tie."""
    rows = close = 0
    if wl.temperature == 0.0:
        for r in requests:
            o = ores[r]
            rows += len(o["argmax"])
            close += int(((o["top1"] - o["top2"]) < NEAR_TIE).sum())
    NEAR_LOG.append(dict(test=label, requests=len(requests), rows=rows, near_rows=close,
                         excused=int(excused)))


def attn_compare(wl, dev, rows=None, nthreads=0):
    out_o, lse_o, st = oracle.attention(wl.cu_nodes, wl.parent, wl.kv_len, wl.slot_base, wl.q,
                                        wl.k_tree, wl.v_tree, wl.k_cache, wl.v_cache, wl.hq,
                                        wl.hkv, oracle.scale_of(wl.head_dim), rows=rows,
                                        nthreads=nthreads)
    assert st == 0
    g_out = dev.out.float().cpu().numpy().reshape(-1, wl.head_dim)
    g_lse = dev.lse.cpu().numpy().reshape(-1)
    if rows is not None:
        rr = np.asarray(rows, dtype=np.int64).reshape(-1, 2)
        idx = rr[:, 0] * wl.hq + rr[:, 1]
        g_out, g_lse = g_out[idx], g_lse[idx]
    err = g_out - out_o
    res = dict(max_abs=float(np.abs(err).max()),
               rel_rms=float(np.sqrt((err ** 2).mean() / (out_o ** 2).mean())),
               lse_err=float(np.abs(g_lse - lse_o).max()), rows=len(out_o))
    assert res["max_abs"] <= ATTN_MAX_ABS, res
    assert res["rel_rms"] <= ATTN_REL_RMS, res
    assert res["lse_err"] <= LSE_ABS, res
    return res


def attn_compare_paged(wl, dev, rows=None, nthreads=0):
    """attn_compare for a DeviceStep on a paged cache: the oracle gathers each request's logical
    cache through the same block table."""
    pc = dev.paged
    out_o, lse_o, st = oracle.attention_paged(wl.cu_nodes, wl.parent, wl.kv_len, pc.block_table,
                                              pc.page_size, wl.q, wl.k_tree, wl.v_tree,
                                              pc.k_pool, pc.v_pool, wl.hq, wl.hkv,
                                              oracle.scale_of(wl.head_dim), rows=rows,
                                              nthreads=nthreads)
    assert st == 0
    g_out = dev.out.float().cpu().numpy().reshape(-1, wl.head_dim)
    g_lse = dev.lse.cpu().numpy().reshape(-1)
    if rows is not None:
        rr = np.asarray(rows, dtype=np.int64).reshape(-1, 2)
        idx = rr[:, 0] * wl.hq + rr[:, 1]
        g_out, g_lse = g_out[idx], g_lse[idx]
    err = g_out - out_o
    res = dict(max_abs=float(np.abs(err).max()),
               rel_rms=float(np.sqrt((err ** 2).mean() / (out_o ** 2).mean())),
               lse_err=float(np.abs(g_lse - lse_o).max()))
    assert res["max_abs"] <= ATTN_MAX_ABS, res
    assert res["rel_rms"] <= ATTN_REL_RMS, res
    assert res["lse_err"] <= LSE_ABS, res
    return res


def compact_compare_paged(wl, dev, ores, requests, excused):
    """Bit-exact check of a paged compaction: the oracle scatters the same accepted rows through
    the block table into a copy of the initial pool; the slots of the checked requests (and
    their kv_len_out) must match."""
    pc = dev.paged
    kpool = oracle._u16(pc.k_pool)[None].copy()
    vpool = oracle._u16(pc.v_pool)[None].copy()
    a = np.zeros(wl.B, dtype=np.int32)
    path = np.full((wl.B, 64), -1, dtype=np.int32)
    path[:, 0] = 0
    for r in requests:
        a[r] = ores[r]["accept_len"]
        path[r] = ores[r]["path"]
    st, newlen = oracle.kv_compact_paged(wl.cu_nodes, wl.kv_len, pc.block_table, pc.page_size,
                                         pc.slot_cap, a, path, oracle._u16(wl.k_tree)[None],
                                         oracle._u16(wl.v_tree)[None], kpool, vpool, 1)
    assert st == 0
    gk = oracle._u16(dev.k_cache.cpu())
    gv = oracle._u16(dev.v_cache.cpu())
    kv_out = dev.kv_len_out.cpu().numpy()
    for r in requests:
        if r in excused:
            continue
        sl = oracle.page_slots(pc.block_table, pc.page_size, r, np.arange(int(newlen[r])))
        assert np.array_equal(gk[sl], kpool[0, sl]) and np.array_equal(gv[sl], vpool[0, sl]), r
        assert kv_out[r] == newlen[r], (r, kv_out[r], newlen[r])


def sample_rows(wl, per_request: int, seed: int = 0):
    """(node, head) pairs: the last node of every request (deepest, all heads of one KV group)
    plus random (node, head) pairs."""
    g = np.random.default_rng(seed)
    rows = []
    G = wl.hq // wl.hkv
    for r in range(wl.B):
        a0, a1 = int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])
        kvh = int(g.integers(wl.hkv))
        for h in range(kvh * G, kvh * G + G):
            rows.append((a1 - 1, h))
        for _ in range(per_request):
            rows.append((int(g.integers(a0, a1)), int(g.integers(wl.hq))))
    return np.asarray(rows, dtype=np.int32)


def greedy_compare(wl, res, requests, nthreads=0):
    """T = 0: per-node argmax / gap and per-request walk outputs.  Returns (excused, near)."""
    ores = oracle.lmhead_accept_many(wl, requests, nthreads=nthreads)
    excused, near = set(), 0
    for r in requests:
        o = ores[r]
        a0, a1 = int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])
        gam = res["node_argmax"][a0:a1]
        gap_o = o["top1"] - o["top2"]
        diff = gam != o["argmax"]
        if diff.any():
            assert (gap_o[diff] < NEAR_TIE).all(), (r, np.nonzero(diff), gap_o[diff])
            excused.add(r)
            near += int(diff.sum())
            continue
        gg = res["node_gap"][a0:a1]
        assert np.all(np.abs(gg - gap_o) <= 1e-3 + 1e-3 * np.abs(gap_o)), (r, gg, gap_o)
        assert res["accept_len"][r] == o["accept_len"], (r, res["accept_len"][r], o["accept_len"])
        assert np.array_equal(res["path"][r], o["path"]), (r, res["path"][r], o["path"])
        assert np.array_equal(res["out_tokens"][r], o["out_tokens"]), r
    return excused, near, ores


def chain_compare(wl, res, requests, nthreads=0):
    """T > 0 chains.  Returns (excused, near)."""
    ores = oracle.lmhead_accept_many(wl, requests, nthreads=nthreads, keep_logits=True)
    excused, near = set(), 0
    T = wl.temperature
    for r in requests:
        o = ores[r]
        a0, a1 = int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])
        ga = int(res["accept_len"][r])
        same = (ga == o["accept_len"] and np.array_equal(res["path"][r], o["path"])
                and np.array_equal(res["out_tokens"][r], o["out_tokens"]))
        if same:
            continue
        z = o["z"] / T
        p = np.exp(z - z.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        qd = wl.q_draft[a0:a1].numpy().astype(np.float64)
        tok = wl.tokens[a0:a1]
        oa = int(o["accept_len"])
        if ga != oa:
            k = min(ga, oa) + 1                       # first node whose decision differs
            U = oracle.uniform(wl.seed, wl.step, r, k, 0, 1)
            pu, qu = p[k - 1, tok[k]], qd[k - 1, tok[k]]
            assert abs(U * qu - pu) <= SAMPLE_REL * max(pu, U * qu), (r, k, U * qu, pu)
        else:
            u = oa
            rejected = o["info"][1] == 1
            _draw_near_tie(wl, r, u, p[u], qd[u], 1.0 if rejected else 0.0,
                           int(res["out_tokens"][r][oa]), int(o["out_tokens"][oa]))
        excused.add(r)
        near += 1
    return excused, near, ores


def race_key(wl, r, u, v, w):
    """The race key log w_v - log(-log U_v) of id v at stop node u, in fp64."""
    U = oracle.uniform(wl.seed, wl.step, r, u, v, 0)
    return np.log(w[v]) - np.log(-np.log(U)) if w[v] > 0 else -np.inf


def _draw_near_tie(wl, r, u, p, q, c, tg, to):
    """The GPU's bonus tg and the oracle's to differ at stop node u: both are winners of the
    exponential race (over max(0, p - c q), or over p when that residual has no positive weight)
    up to fp32 rounding.  The GPU forms each weight in fp32 from fp32 logits: p with a relative
    error of a few 1e-7, and p - c q with an absolute error of a few 1e-7 (p + c q).  So the two
    ids' fp64 keys must agree within SAMPLE_REL plus that weight error over the weight, and an id
    the fp64 weights exclude must have its weight within that error of zero."""
    w = np.maximum(p - c * q, 0.0) if c > 0 else p.copy()
    if c > 0 and not (w > 0).any():
        w = p.copy()
        c = 0.0
    err = 4e-6 * (p + c * q)

    def tol(v):
        return SAMPLE_REL + (err[v] / w[v] if w[v] > 0 else np.inf)

    if w[tg] <= 0:                                 # the GPU saw a weight the fp64 side rounds to 0
        assert abs(p[tg] - c * q[tg]) <= err[tg], (r, tg, to, p[tg], q[tg], c)
        return
    kg, ko = race_key(wl, r, u, tg, w), race_key(wl, r, u, to, w)
    assert kg <= ko and ko - kg <= tol(tg) + tol(to), (r, tg, to, kg, ko)


def tree_compare(wl, res, requests, nthreads=0):
    """T > 0 on branching trees: the GPU's walk against the oracle's.  Where they differ, the
    first differing decision is replayed in fp64 and must be a sampling near-tie: an accept test
    U q(x) vs r(x) = max(0, p(x) - c q(x)) / N(c), or the bonus draw.  Returns (excused, near)."""
    ores = oracle.lmhead_accept_many(wl, requests, nthreads=nthreads, keep_logits=True)
    excused, near = set(), 0
    T = wl.temperature
    for r in requests:
        o = ores[r]
        a0, a1 = int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])
        n = a1 - a0
        ga, oa = int(res["accept_len"][r]), int(o["accept_len"])
        if (ga == oa and np.array_equal(res["path"][r], o["path"])
                and np.array_equal(res["out_tokens"][r], o["out_tokens"])):
            continue
        z = o["z"] / T
        p = np.exp(z - z.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        qd = wl.q_draft[a0:a1].numpy().astype(np.float64)
        par = wl.parent[a0:a1]
        tok = wl.tokens[a0:a1]
        gp, op = list(res["path"][r][:ga + 1]), list(o["path"][:oa + 1])
        u, depth, settled = 0, 0, False
        while not settled:
            gnext = gp[depth + 1] if depth + 1 <= ga else None
            onext = op[depth + 1] if depth + 1 <= oa else None
            c, N = 0.0, 1.0
            for j in [j for j in range(1, n) if par[j] == u]:
                x = int(tok[j])
                U = oracle.uniform(wl.seed, wl.step, r, j, 0, 1)
                uq, rx = U * qd[u, x], max(0.0, p[u, x] - c * qd[u, x]) / N
                if (onext == j) != (gnext == j):
                    assert abs(uq - rx) <= SAMPLE_REL * max(uq, rx), (r, u, j, uq, rx)
                    settled = True
                    break
                if onext == j:
                    break
                c += N
                N = np.maximum(p[u] - c * qd[u], 0.0).sum()
            if settled:
                break
            if onext is None and gnext is None:        # same path, different bonus
                _draw_near_tie(wl, r, u, p[u], qd[u], c, int(res["out_tokens"][r][ga]),
                               int(o["out_tokens"][oa]))
                break
            assert onext == gnext, (r, gp, op)
            u, depth = onext, depth + 1
        excused.add(r)
        near += 1
    return excused, near, ores


def compact_compare(wl, dev, ores, requests, excused):
    """Bit-exact check of the compacted rows of each request against the oracle's compaction
    of that request's slot range (single layer)."""
    kc = dev.k_cache
    vc = dev.v_cache
    kv_out = dev.kv_len_out.cpu().numpy()
    for r in requests:
        if r in excused:
            continue
        o = ores[r]
        a = int(o["accept_len"])
        base, cap = int(wl.slot_base[r]), int(wl.slot_cap[r])
        a0, a1 = int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])
        sub_k = oracle._u16(wl.k_cache[base:base + cap]).copy()
        sub_v = oracle._u16(wl.v_cache[base:base + cap]).copy()
        cu = np.array([0, a1 - a0], dtype=np.int32)
        path = o["path"].reshape(1, 64)
        st, newlen = oracle.kv_compact(cu, wl.kv_len[r:r + 1], np.zeros(1, np.int64),
                                       wl.slot_cap[r:r + 1], np.array([a], np.int32), path,
                                       wl.k_tree[a0:a1], wl.v_tree[a0:a1], sub_k, sub_v, 1,
                                       (a1 - a0) * wl.hkv * wl.head_dim,
                                       cap * wl.hkv * wl.head_dim, wl.hkv, wl.head_dim)
        assert st == 0
        gk = oracle._u16(kc[base:base + cap].cpu())
        gv = oracle._u16(vc[base:base + cap].cpu())
        assert np.array_equal(gk, sub_k), r
        assert np.array_equal(gv, sub_v), r
        assert kv_out[r] == newlen[0], (r, kv_out[r], newlen[0])


# Rounding bounds of the low-rank head's GPU arithmetic (u: unit roundoff).
U_BF16 = 2.0 ** -8          # bf16 keeps 8 significant bits: |bf16(x) - x| <= 2^-8 |x|
U_FP32 = 2.0 ** -24


def _gamma(n):
    """Worst-case relative error bound of an n-term fp32 sum of products, n u / (1 - n u)."""
    return n * U_FP32 / (1.0 - n * U_FP32)


def _bf16_f32(x):
    u = oracle._u16(x)
    return np.frombuffer((u.astype(np.uint32) << 16).tobytes(), np.float32).reshape(u.shape)


def lowrank_bounds(lw, g):
    """Per (row, id) bound on |z~_gpu - z~|, and a function giving the bound on the exact logit's
    error of (row, id).

    The library computes g = h D^T with fp32 accumulation over H terms (error e <= gamma_H
    sum |h||D|), rounds it to bf16 (the screen GEMM's operand type: a further 2^-8 |g_gpu|), and
    the screen z~ = bf16(g) U^T with fp32 accumulation over r terms.  So
        |z~_gpu - z~| <= sum_j |dg_j| |U_vj| + gamma_r sum_j (|g_j| + |dg_j|) |U_vj|,
        |dg_j| <= 2^-8 (|g_j| + e_j) + e_j.
    The exact logits h . W_c accumulate H fp32 products: error <= gamma_H sum |h| |W_c|.
    (The bounds themselves are evaluated in fp32: they need no more.)"""
    h = np.abs(_bf16_f32(lw.hidden))
    e = _gamma(lw.H) * (h @ np.abs(_bf16_f32(lw.D)).T)
    ag = np.abs(g).astype(np.float32)
    dg = (U_BF16 * (ag + e) + e).astype(np.float32)
    aU = np.abs(_bf16_f32(lw.U)).T
    screen = dg @ aU + np.float32(_gamma(lw.r)) * ((ag + dg) @ aU)
    wb = oracle._u16(lw.W)

    def exact(m, c):
        wc = np.frombuffer((wb[c].astype(np.uint32) << 16).tobytes(), np.float32)
        return _gamma(lw.H) * float(h[m] @ np.abs(wc))

    return screen.astype(np.float64), exact


def lowrank_compare(lw, ids, logit, nthreads=0):
    """The GPU's candidates against the oracle's.  Candidate sets must agree except for ids that
    the screen's rounding bound (lowrank_bounds) allows across the cut: an id in one set only
    must have an exact screen value within its bound plus the bound of the oracle's k-th
    candidate of the k-th value.  Exact logits of common ids agree within their fp32 bound, and
    the order by exact logit agrees except between candidates whose fp64 logits are within the
    sum of their bounds.  Returns the number of rows with a set difference."""
    oid, olg, kth, za, g = oracle.lowrank_candidates(lw.hidden, lw.D, lw.U, lw.W, lw.k,
                                                     keep_approx=True, keep_g=True,
                                                     nthreads=nthreads)
    screen, exact = lowrank_bounds(lw, g)
    differ = 0
    for m in range(lw.M):
        sg, so = set(ids[m].tolist()), set(oid[m].tolist())
        kid = min(so, key=lambda c: (za[m, c], -c))      # the oracle's k-th candidate
        for c in sg ^ so:
            assert 0 <= c < lw.V, (m, c)
            assert abs(za[m, c] - kth[m]) <= screen[m, c] + screen[m, kid], \
                (m, c, za[m, c], kth[m], screen[m, c], screen[m, kid])
        differ += int(sg != so)
        o_of = dict(zip(oid[m].tolist(), olg[m].tolist()))
        for i, c in enumerate(ids[m].tolist()):
            if c in o_of:
                z = o_of[c]
                assert abs(logit[m, i] - z) <= exact(m, c) + 1e-6, (m, c, logit[m, i], z)
        # ordering: consecutive GPU entries that are both oracle candidates keep the oracle order
        # unless their fp64 logits are within the sum of their bounds
        common = [c for c in ids[m].tolist() if c in o_of]
        for a, b in zip(common, common[1:]):
            za_, zb_ = o_of[a], o_of[b]
            assert za_ > zb_ or abs(za_ - zb_) <= exact(m, a) + exact(m, b) or \
                (za_ == zb_ and a < b), (m, a, b, za_, zb_)
    return differ
