"""fp64 CPU oracle for draft-tree verification -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import
this package.  The product path (the CUDA library and its Python binding) never does: it shares no
code with this module, and this module imports nothing from it.

Every function is a thin ctypes marshaller around the plain C definitions in ``oracle.c``; the
per-request composition below only slices rows and calls those definitions in order, and the
paged-cache forms first gather (or scatter) rows through the block tables with numpy indexing.
"""
from __future__ import annotations

import ctypes as C

import numpy as np

from . import _build

_lib = None

I32P = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
I64P = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
U64P = np.ctypeslib.ndpointer(np.uint64, flags="C_CONTIGUOUS")
U16P = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
F64P = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
F32P = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")

OK, EINVAL, EUNSUPPORTED, ENOSPACE = 0, -1, -2, -6


def _bind(path: str):
    """Load the oracle library at `path` and declare its signatures."""
    L = C.CDLL(path)
    L.oracle_max_threads.restype = C.c_int
    L.oracle_ancestry.argtypes = [C.c_int, I32P, U64P, I32P]
    L.oracle_ancestry.restype = C.c_int
    L.oracle_attention.argtypes = [C.c_int, I32P, I32P, I32P, I64P, U16P, U16P, U16P, U16P,
                                   U16P, C.c_int, C.c_int, C.c_int, C.c_double, C.c_int,
                                   C.c_void_p, F64P, F64P, C.c_int]
    L.oracle_attention.restype = C.c_int
    L.oracle_logits.argtypes = [C.c_int, I32P, C.c_int, C.c_int, U16P, U16P, F64P, C.c_int]
    L.oracle_logits.restype = None
    L.oracle_row_top2.argtypes = [C.c_int, C.c_int, F64P, I32P, F64P, F64P]
    L.oracle_row_top2.restype = None
    L.oracle_walk_greedy.argtypes = [C.c_int, I32P, I32P, I32P, I32P, I32P]
    L.oracle_walk_greedy.restype = C.c_int
    L.oracle_philox4x64.argtypes = [U64P, U64P, U64P]
    L.oracle_philox4x64.restype = None
    L.oracle_uniform.argtypes = [C.c_uint64, C.c_uint64, C.c_uint32, C.c_uint32, C.c_uint32,
                                 C.c_uint32]
    L.oracle_uniform.restype = C.c_double
    L.oracle_race.argtypes = [C.c_int, F64P, C.c_uint64, C.c_uint64, C.c_int, C.c_int,
                              C.POINTER(C.c_double)]
    L.oracle_race.restype = C.c_int
    L.oracle_accept_chain.argtypes = [C.c_int, I32P, I32P, F64P, F32P, C.c_int, C.c_double,
                                      C.c_uint64, C.c_uint64, C.c_int, I32P, I32P, I32P]
    L.oracle_accept_chain.restype = C.c_int
    L.oracle_kv_compact.argtypes = [C.c_int, I32P, I32P, I64P, I32P, I32P, I32P, U16P, U16P,
                                    U16P, U16P, C.c_int, C.c_int64, C.c_int64, C.c_int,
                                    C.c_int, I32P]
    L.oracle_kv_compact.restype = C.c_int
    L.oracle_accept_chain_batch.argtypes = [C.c_int, I32P, I32P, I32P, F64P, F32P, C.c_int,
                                            C.c_double, C.c_uint64, C.c_uint64, I32P, I32P,
                                            I32P, I32P, C.c_int]
    L.oracle_accept_chain_batch.restype = None
    L.oracle_accept_tree.argtypes = [C.c_int, I32P, I32P, F64P, F32P, C.c_int, C.c_double,
                                     C.c_uint64, C.c_uint64, C.c_int, I32P, I32P, I32P,
                                     C.POINTER(C.c_double)]
    L.oracle_accept_tree.restype = C.c_int
    L.oracle_accept_tree_batch.argtypes = [C.c_int, I32P, I32P, I32P, F64P, F32P, C.c_int,
                                           C.c_double, C.c_uint64, C.c_uint64, I32P, I32P,
                                           I32P, I32P, F64P, C.c_int]
    L.oracle_accept_tree_batch.restype = None
    L.oracle_bf16_round.argtypes = [C.c_double]
    L.oracle_bf16_round.restype = C.c_uint16
    L.oracle_lowrank_candidates.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                            U16P, U16P, U16P, U16P, I32P, F64P, C.c_void_p,
                                            C.c_void_p, C.c_void_p, C.c_int]
    L.oracle_lowrank_candidates.restype = None
    L.oracle_race_many.argtypes = [C.c_int, C.c_int, F64P, C.c_uint64, C.c_uint64, C.c_int,
                                   C.c_int, I32P, C.c_int]
    L.oracle_race_many.restype = None
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = _bind(_build.build())
    return _lib


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def _u16(x) -> np.ndarray:
    """uint16 bits of a bf16 torch tensor or a uint16 numpy array (no copy when contiguous)."""
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x, dtype=np.uint16)
    import torch
    t = x.detach().cpu().contiguous()
    assert t.dtype == torch.bfloat16
    return t.view(torch.int16).numpy().view(np.uint16)


def _i32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x), dtype=np.int32)


# ------------------------------------------------------------------------------------ primitives
def ancestry(parent):
    parent = _i32(parent)
    n = len(parent)
    anc = np.zeros(max(n, 1), dtype=np.uint64)
    dep = np.zeros(max(n, 1), dtype=np.int32)
    st = lib().oracle_ancestry(n, parent, anc, dep)
    return st, anc[:n], dep[:n]


def attention(cu_nodes, parent, kv_len, slot_base, q, k_tree, v_tree, k_cache, v_cache, hq, hkv,
              scale, rows=None, nthreads=0):
    """(out [k, d] fp64, lse [k] fp64, status) for the listed (node, head) rows, or all rows."""
    cu = _i32(cu_nodes)
    B = len(cu) - 1
    qn = _u16(q)
    d = qn.shape[-1] if qn.ndim > 1 else 128
    if rows is None:
        nrows, rp, count = 0, None, int(cu[-1]) * hq
    else:
        rr = _i32(rows).reshape(-1, 2)
        nrows, rp, count = len(rr), rr.ctypes.data_as(C.c_void_p), len(rr)
    out = np.zeros((max(count, 1), d), dtype=np.float64)
    lse = np.zeros(max(count, 1), dtype=np.float64)
    st = lib().oracle_attention(B, cu, _i32(parent), _i32(kv_len),
                                np.ascontiguousarray(slot_base, dtype=np.int64), qn.reshape(-1),
                                _u16(k_tree).reshape(-1), _u16(v_tree).reshape(-1),
                                _u16(k_cache).reshape(-1), _u16(v_cache).reshape(-1), hq, hkv, d,
                                float(scale), nrows, rp, out, lse, int(nthreads))
    return out[:count], lse[:count], st


def logits(hidden, w, rows, nthreads=0):
    hn = _u16(hidden)
    wn = _u16(w)
    H = wn.shape[1]
    V = wn.shape[0]
    rows = _i32(rows)
    z = np.empty((len(rows), V), dtype=np.float64)
    if len(rows):
        lib().oracle_logits(len(rows), rows, H, V, hn.reshape(-1), wn.reshape(-1), z,
                            int(nthreads))
    return z


def row_top2(z):
    z = np.ascontiguousarray(z, dtype=np.float64)
    n, V = z.shape
    arg = np.empty(n, dtype=np.int32)
    t1 = np.empty(n, dtype=np.float64)
    t2 = np.empty(n, dtype=np.float64)
    if n:
        lib().oracle_row_top2(n, V, z, arg, t1, t2)
    return arg, t1, t2


def walk_greedy(parent, tokens, arg):
    path = np.empty(64, dtype=np.int32)
    out = np.empty(65, dtype=np.int32)
    a = lib().oracle_walk_greedy(len(parent), _i32(parent), _i32(tokens), _i32(arg), path, out)
    return a, path, out


def philox4x64(ctr, key):
    out = np.empty(4, dtype=np.uint64)
    lib().oracle_philox4x64(np.ascontiguousarray(ctr, dtype=np.uint64),
                            np.ascontiguousarray(key, dtype=np.uint64), out)
    return out


def uniform(seed, step, r, node, v, stream):
    return float(lib().oracle_uniform(seed, step, r, node, v, stream))


def race(w, seed, step, r, node):
    w = np.ascontiguousarray(w, dtype=np.float64)
    bk = C.c_double()
    tok = lib().oracle_race(len(w), w, seed, step, r, node, C.byref(bk))
    return tok, bk.value


def accept_chain(parent, tokens, z, q, T, seed, step, r):
    z = np.ascontiguousarray(z, dtype=np.float64)
    q = np.ascontiguousarray(q, dtype=np.float32)
    n, V = z.shape
    path = np.empty(64, dtype=np.int32)
    out = np.empty(65, dtype=np.int32)
    info = np.zeros(3, dtype=np.int32)
    a = lib().oracle_accept_chain(n, _i32(parent), _i32(tokens), z, q, V, float(T), seed, step,
                                  r, path, out, info)
    return a, path, out, info


def accept_chain_batch(cu_nodes, parent, tokens, z, q, T, seed, step, nthreads=0):
    """Batched oracle_accept_chain; returns (accept_len [B], path [B,64], out [B,65], info [B,3])."""
    cu = _i32(cu_nodes)
    B = len(cu) - 1
    z = np.ascontiguousarray(z, dtype=np.float64)
    q = np.ascontiguousarray(q, dtype=np.float32)
    V = z.shape[1]
    a = np.empty(B, dtype=np.int32)
    path = np.empty((B, 64), dtype=np.int32)
    out = np.empty((B, 65), dtype=np.int32)
    info = np.zeros((B, 3), dtype=np.int32)
    lib().oracle_accept_chain_batch(B, cu, _i32(parent), _i32(tokens), z.reshape(-1),
                                    q.reshape(-1), V, float(T), seed, step, a, path.reshape(-1),
                                    out.reshape(-1), info.reshape(-1), int(nthreads))
    return a, path, out, info


def accept_tree(parent, tokens, z, q, T, seed, step, r):
    """Multi-candidate acceptance over one request's tree; returns (a, path, out, info, c)."""
    z = np.ascontiguousarray(z, dtype=np.float64)
    q = np.ascontiguousarray(q, dtype=np.float32)
    n, V = z.shape
    path = np.empty(64, dtype=np.int32)
    out = np.empty(65, dtype=np.int32)
    info = np.zeros(3, dtype=np.int32)
    c = C.c_double()
    a = lib().oracle_accept_tree(n, _i32(parent), _i32(tokens), z, q, V, float(T), seed, step, r,
                                 path, out, info, C.byref(c))
    return a, path, out, info, c.value


def accept_tree_batch(cu_nodes, parent, tokens, z, q, T, seed, step, nthreads=0):
    """Batched oracle_accept_tree; returns (accept_len [B], path [B,64], out [B,65], info [B,3],
    c [B])."""
    cu = _i32(cu_nodes)
    B = len(cu) - 1
    z = np.ascontiguousarray(z, dtype=np.float64)
    q = np.ascontiguousarray(q, dtype=np.float32)
    V = z.shape[1]
    a = np.empty(B, dtype=np.int32)
    path = np.empty((B, 64), dtype=np.int32)
    out = np.empty((B, 65), dtype=np.int32)
    info = np.zeros((B, 3), dtype=np.int32)
    c = np.zeros(B, dtype=np.float64)
    lib().oracle_accept_tree_batch(B, cu, _i32(parent), _i32(tokens), z.reshape(-1),
                                   q.reshape(-1), V, float(T), seed, step, a, path.reshape(-1),
                                   out.reshape(-1), info.reshape(-1), c, int(nthreads))
    return a, path, out, info, c


def race_many(w, n, seed, step, r0, node, nthreads=0):
    w = np.ascontiguousarray(w, dtype=np.float64)
    out = np.empty(n, dtype=np.int32)
    lib().oracle_race_many(n, len(w), w, seed, step, r0, node, out, int(nthreads))
    return out


def kv_compact(cu_nodes, kv_len, slot_base, slot_cap, accept_len, path, k_tree, v_tree, k_cache,
               v_cache, n_layers, tree_layer_stride, cache_layer_stride, hkv, d):
    """Compacts in place into the given uint16 caches; returns (status, kv_len_out)."""
    cu = _i32(cu_nodes)
    B = len(cu) - 1
    out = np.empty(B, dtype=np.int32)
    kc = k_cache if isinstance(k_cache, np.ndarray) else _u16(k_cache)
    vc = v_cache if isinstance(v_cache, np.ndarray) else _u16(v_cache)
    st = lib().oracle_kv_compact(B, cu, _i32(kv_len), np.ascontiguousarray(slot_base, np.int64),
                                 _i32(slot_cap), _i32(accept_len),
                                 _i32(path).reshape(-1), _u16(k_tree).reshape(-1),
                                 _u16(v_tree).reshape(-1), kc.reshape(-1), vc.reshape(-1),
                                 n_layers, tree_layer_stride, cache_layer_stride, hkv, d, out)
    return st, out


def bf16_round(x) -> int:
    return int(lib().oracle_bf16_round(float(x)))


def lowrank_candidates(hidden, D, U, W, k, keep_approx=False, nthreads=0, keep_g=False):
    """The low-rank candidate head over the rows of `hidden`: returns (ids [M,k], exact logits
    [M,k], k-th approximate logit [M], approximate logits [M,V] or None), plus the down
    projection g [M,r] when keep_g."""
    h, d, u, w = _u16(hidden), _u16(D), _u16(U), _u16(W)
    M, H = h.shape
    r, V = d.shape[0], u.shape[0]
    ids = np.empty((M, k), dtype=np.int32)
    lg = np.empty((M, k), dtype=np.float64)
    kth = np.empty(M, dtype=np.float64)
    za = np.empty((M, V), dtype=np.float64) if keep_approx else None
    g = np.empty((M, r), dtype=np.float64) if keep_g else None
    lib().oracle_lowrank_candidates(M, H, V, r, k, h.reshape(-1), d.reshape(-1), u.reshape(-1),
                                    w.reshape(-1), ids.reshape(-1), lg.reshape(-1),
                                    kth.ctypes.data_as(C.c_void_p),
                                    za.ctypes.data_as(C.c_void_p) if keep_approx else None,
                                    g.ctypes.data_as(C.c_void_p) if keep_g else None,
                                    int(nthreads))
    if keep_g:
        return ids, lg, kth, za, g
    return ids, lg, kth, za


# ------------------------------------------------------------------------------- paged caches
# A paged cache holds each request's positions in fixed-size pages of a shared pool: logical
# position t of request r lives at pool slot block_table[r, t // P] * P + t % P (pool arrays
# [num_pages * P][hkv][d]).  The oracle's paged calls are the contiguous definitions applied to
# the logical caches gathered through the block tables (a plain index gather).

def page_slots(block_table, page_size, r, t):
    """Pool slots of logical positions t (array) of request r."""
    t = np.asarray(t, dtype=np.int64)
    return np.asarray(block_table)[r, t // page_size].astype(np.int64) * page_size + t % page_size


def attention_paged(cu_nodes, parent, kv_len, block_table, page_size, q, k_tree, v_tree, k_pool,
                    v_pool, hq, hkv, scale, rows=None, nthreads=0):
    """Tree attention over a paged cache: each request's first kv_len[r] positions are gathered
    through its block table into a contiguous cache, then `attention` runs on it."""
    kp, vp = _u16(k_pool), _u16(v_pool)
    B = len(kv_len)
    base = np.zeros(B, dtype=np.int64)
    ks, vs = [], []
    off = 0
    for r in range(B):
        sl = page_slots(block_table, page_size, r, np.arange(int(kv_len[r])))
        ks.append(kp[sl])
        vs.append(vp[sl])
        base[r] = off
        off += int(kv_len[r])
    kc = np.concatenate(ks) if off else np.zeros((1,) + kp.shape[1:], np.uint16)
    vc = np.concatenate(vs) if off else np.zeros((1,) + vp.shape[1:], np.uint16)
    return attention(cu_nodes, parent, kv_len, base, q, k_tree, v_tree, kc, vc, hq, hkv, scale,
                     rows=rows, nthreads=nthreads)


def kv_compact_paged(cu_nodes, kv_len, block_table, page_size, slot_cap, accept_len, path,
                     k_tree, v_tree, k_pool, v_pool, n_layers):
    """Compaction into a paged cache, in place on the uint16 pools [n_layers][slots][hkv][d]:
    pool[slot(kv_len[r] + k)] <- tree[cu_nodes[r] + path[r][k]], k = 0..a.  A request whose
    rows would pass slot_cap[r] is left untouched.  Returns (status, kv_len_out)."""
    cu = _i32(cu_nodes)
    B = len(cu) - 1
    kt, vt = _u16(k_tree), _u16(v_tree)
    out = np.asarray(kv_len, dtype=np.int32).copy()
    status = 0
    for r in range(B):
        n = int(cu[r + 1] - cu[r])
        a, L = int(accept_len[r]), int(kv_len[r])
        pr = np.asarray(path)[r, :a + 1]
        if n < 1 or a < 0 or a >= n or (pr < 0).any() or (pr >= n).any():
            status = status or EINVAL
            continue
        if L + a + 1 > int(slot_cap[r]):
            status = status or ENOSPACE
            continue
        dst = page_slots(block_table, page_size, r, np.arange(L, L + a + 1))
        src = int(cu[r]) + pr
        for layer in range(n_layers):
            k_pool[layer, dst] = kt[layer, src]
            v_pool[layer, dst] = vt[layer, src]
        out[r] = L + a + 1
    return status, out


# --------------------------------------------------------------------------- per-request passes
def lmhead_accept(wl, requests=None, nthreads=0, keep_logits=False):
    """The oracle's LM head + acceptance for the listed requests of a Workload.

    Returns a dict of per-request results: accept_len, path [64], out_tokens [65], and for T=0
    per-node argmax, top1, top2; for T>0 the stop node / rejection / fallback info.
    """
    reqs = range(wl.B) if requests is None else requests
    res = {}
    for r in reqs:
        a0, a1 = int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])
        rows = np.arange(a0, a1, dtype=np.int32)
        z = logits(wl.hidden, wl.w_lm, rows, nthreads)
        par = wl.parent[a0:a1]
        tok = wl.tokens[a0:a1]
        if wl.temperature == 0.0:
            arg, t1, t2 = row_top2(z)
            a, path, out = walk_greedy(par, tok, arg)
            res[r] = dict(accept_len=a, path=path, out_tokens=out, argmax=arg, top1=t1, top2=t2)
        else:
            qd = wl.q_draft[a0:a1].numpy()
            if np.array_equal(par, np.arange(-1, a1 - a0 - 1)):
                a, path, out, info = accept_chain(par, tok, z, qd, wl.temperature, wl.seed,
                                                  wl.step, r)
                c = 1.0 if info[1] else 0.0
            else:
                a, path, out, info, c = accept_tree(par, tok, z, qd, wl.temperature, wl.seed,
                                                    wl.step, r)
            res[r] = dict(accept_len=a, path=path, out_tokens=out, info=info, c=c,
                          z=z if keep_logits else None)
    return res


def lmhead_accept_many(wl, requests=None, nthreads=0, keep_logits=False, chunk_rows=512):
    """lmhead_accept for many requests at once: the logits of up to chunk_rows node rows come
    from one oracle_logits call (one pass over the head per chunk instead of one per request);
    the per-request definitions that follow are the same calls as in lmhead_accept."""
    reqs = list(range(wl.B) if requests is None else requests)
    res = {}
    i = 0
    while i < len(reqs):
        group, nrow = [], 0
        while i < len(reqs) and (not group or nrow + wl.nodes(reqs[i]) <= chunk_rows):
            group.append(reqs[i])
            nrow += wl.nodes(reqs[i])
            i += 1
        rows = np.concatenate([np.arange(int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1]),
                                         dtype=np.int32) for r in group])
        zall = logits(wl.hidden, wl.w_lm, rows, nthreads)
        off = 0
        for r in group:
            a0, a1 = int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])
            z = zall[off:off + a1 - a0]
            off += a1 - a0
            par = wl.parent[a0:a1]
            tok = wl.tokens[a0:a1]
            if wl.temperature == 0.0:
                arg, t1, t2 = row_top2(z)
                a, path, out = walk_greedy(par, tok, arg)
                res[r] = dict(accept_len=a, path=path, out_tokens=out, argmax=arg, top1=t1,
                              top2=t2)
            else:
                qd = wl.q_draft[a0:a1].numpy()
                if np.array_equal(par, np.arange(-1, a1 - a0 - 1)):
                    a, path, out, info = accept_chain(par, tok, z, qd, wl.temperature, wl.seed,
                                                      wl.step, r)
                    c = 1.0 if info[1] else 0.0
                else:
                    a, path, out, info, c = accept_tree(par, tok, z, qd, wl.temperature,
                                                        wl.seed, wl.step, r)
                res[r] = dict(accept_len=a, path=path, out_tokens=out, info=info, c=c,
                              z=z.copy() if keep_logits else None)
    return res


def row_argmax(hidden, w, nthreads=0, chunk_rows=512):
    """Each hidden row's argmax of hidden . w^T (fp64, lowest id on ties)."""
    n = int(hidden.shape[0])
    out = np.empty(n, dtype=np.int32)
    for i in range(0, n, chunk_rows):
        rows = np.arange(i, min(n, i + chunk_rows), dtype=np.int32)
        out[i:i + len(rows)] = row_top2(logits(hidden, w, rows, nthreads))[0]
    return out


def scale_of(head_dim: int) -> float:
    return 1.0 / float(np.sqrt(head_dim))

