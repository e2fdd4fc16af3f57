"""Comparisons of the CUDA path against the fp64 oracle (test infrastructure).

Tolerances:
* attention output: max-abs <= 2e-2 and relative RMS <= 5e-3 against fp64 (bf16 inputs and
  output, fp32 accumulation); lse: |err| <= 1e-3 (fp32 softmax statistics over <= 131k keys);
* argmax, paths, accept lengths, bonus tokens, compacted KV: bit-exact, except at logit near-ties
  (fp64 top1 - top2 < 1e-3), which are logged and counted and excuse the rest of that request;
* per-node top1-top2 gap: |err| <= 1e-3 + 1e-3 |gap| (fp32 accumulation over hidden_dim);
* T > 0: accept decisions and drawn tokens bit-exact, except sampling near-ties where the fp64
  quantities compared differ by less than 1e-5 relative (fp32 vs fp64 rounding): U*q vs p for
  an accept test, the two blocks' race keys, or the inverse-CDF threshold inside a block.
"""
from __future__ import annotations

import numpy as np

import oracle

ATTN_MAX_ABS = 2e-2
ATTN_REL_RMS = 5e-3
LSE_ABS = 1e-3
NEAR_TIE = 1e-3
SAMPLE_REL = 1e-5


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
    ores = oracle.lmhead_accept(wl, requests, nthreads=nthreads)
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
    ores = oracle.lmhead_accept(wl, requests, nthreads=nthreads, keep_logits=True)
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
            tg, to = int(res["out_tokens"][r][oa]), int(o["out_tokens"][oa])
            rejected = o["info"][1] == 1
            w = np.maximum(p[u] - qd[u], 0.0) if rejected else p[u].copy()
            if rejected and not (w > 0).any():
                w = p[u].copy()
            V = len(w)
            bg, bo = tg // 128, to // 128

            def bkey(b):
                Wb = w[b * 128:(b + 1) * 128].sum()
                Ub = oracle.uniform(wl.seed, wl.step, r, u, b, 2)
                return np.log(Wb) - np.log(-np.log(Ub)) if Wb > 0 else -np.inf

            if bg != bo:
                kg, ko = bkey(bg), bkey(bo)
                assert np.isfinite(kg) and abs(kg - ko) <= SAMPLE_REL * max(1.0, abs(ko)), \
                    (r, tg, to, kg, ko)
            else:
                blk = w[bo * 128:min(V, (bo + 1) * 128)]
                c = np.cumsum(blk)
                W = c[-1]
                thr = oracle.uniform(wl.seed, wl.step, r, u, bo, 3) * W
                i = tg - bo * 128
                before = c[i - 1] if i > 0 else 0.0
                assert blk[i] > 0 and c[i] > thr - SAMPLE_REL * W and \
                    before <= thr + SAMPLE_REL * W, (r, tg, to, c[i], before, thr, W)
        excused.add(r)
        near += 1
    return excused, near, ores


def _draw_near_tie(wl, r, u, w, tg, to):
    """The GPU's bonus tg and the oracle's to differ at stop node u with weights w: the two
    blocks' race keys, or the inverse-CDF threshold inside the common block, must be within
    rounding."""
    bg, bo = tg // 128, to // 128

    def bkey(b):
        Wb = w[b * 128:(b + 1) * 128].sum()
        Ub = oracle.uniform(wl.seed, wl.step, r, u, b, 2)
        return np.log(Wb) - np.log(-np.log(Ub)) if Wb > 0 else -np.inf

    if bg != bo:
        kg, ko = bkey(bg), bkey(bo)
        assert np.isfinite(kg) and abs(kg - ko) <= SAMPLE_REL * max(1.0, abs(ko)), \
            (r, tg, to, kg, ko)
    else:
        blk = w[bo * 128:min(len(w), (bo + 1) * 128)]
        c = np.cumsum(blk)
        W = c[-1]
        thr = oracle.uniform(wl.seed, wl.step, r, u, bo, 3) * W
        i = tg - bo * 128
        before = c[i - 1] if i > 0 else 0.0
        assert blk[i] > 0 and c[i] > thr - SAMPLE_REL * W and before <= thr + SAMPLE_REL * W, \
            (r, tg, to, c[i], before, thr, W)


def tree_compare(wl, res, requests, nthreads=0):
    """T > 0 on branching trees: the GPU's walk against the oracle's.  Where they differ, the
    first differing decision is replayed in fp64 and must be a sampling near-tie: an accept test
    U q(x) vs r(x) = max(0, p(x) - c q(x)) / N(c), or the bonus draw.  Returns (excused, near)."""
    ores = oracle.lmhead_accept(wl, requests, nthreads=nthreads, keep_logits=True)
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
                w = np.maximum(p[u] - c * qd[u], 0.0)
                _draw_near_tie(wl, r, u, w, int(res["out_tokens"][r][ga]),
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


LR_SCREEN_TOL = 1e-3    # |z~ - k-th z~| allowed for a candidate-set difference (g's bf16 rounding)


def lowrank_compare(lw, ids, logit, nthreads=0):
    """The GPU's candidates against the oracle's.  Candidate sets must agree except for ids whose
    approximate logit lies within LR_SCREEN_TOL (1 + |k-th|) of the k-th (the screen's operand g is
    bf16, so fp32-vs-fp64 rounding of g can move such ids across the cut); exact logits of common
    ids within 1e-3 (1 + |z|); the order by exact logit must agree except between candidates whose
    fp64 logits differ by less than 1e-3.  Returns the number of rows with a set difference."""
    oid, olg, kth, za = oracle.lowrank_candidates(lw.hidden, lw.D, lw.U, lw.W, lw.k,
                                                  keep_approx=True, nthreads=nthreads)
    differ = 0
    for m in range(lw.M):
        sg, so = set(ids[m].tolist()), set(oid[m].tolist())
        tol = LR_SCREEN_TOL * (1.0 + abs(kth[m]))
        for c in sg ^ so:
            assert 0 <= c < lw.V and abs(za[m, c] - kth[m]) <= tol, (m, c, za[m, c], kth[m])
        differ += int(sg != so)
        o_of = dict(zip(oid[m].tolist(), olg[m].tolist()))
        for i, c in enumerate(ids[m].tolist()):
            if c in o_of:
                z = o_of[c]
                assert abs(logit[m, i] - z) <= 1e-3 * (1.0 + abs(z)), (m, c, logit[m, i], z)
        # ordering: consecutive GPU entries that are both oracle candidates keep the oracle order
        # unless their fp64 logits are within 1e-3
        common = [c for c in ids[m].tolist() if c in o_of]
        for a, b in zip(common, common[1:]):
            za_, zb_ = o_of[a], o_of[b]
            assert za_ > zb_ or abs(za_ - zb_) < 1e-3 or (za_ == zb_ and a < b), (m, a, b, za_, zb_)
    return differ
