"""Seeded synthetic workloads for draft-tree verification.

This module only *constructs inputs*: trees, draft tokens, activations, weights, KV caches and
draft distributions.  It holds none of the verification arithmetic (no attention, no LM head, no
acceptance rule), so both the CUDA library and the fp64 oracle can consume what it makes without
sharing any of the method's code.

Shapes follow the workloads of the EAGLE-4 pages (single request up to 512 concurrent, trees of
4-64 nodes, 27B-class dense target: hidden 5120, 40 query heads / 8 KV heads, head_dim 128,
vocab 151936).  The synthetic recipe and every reading it takes are listed in the design notes:

* bf16 tensors are fp32 normal samples rounded to nearest-even; "N(0,s)" reads as sigma = s.
* trees: a spine down to the depth cap, the remaining nodes attached to uniformly random eligible
  parents (depth, branching and per-level width caps), then relabelled in BFS order so that
  parent[i] < i.  Node 0 is the root (the last committed token).
* T=0 draft tokens: every node u gets a planted target token t*_u; its hidden state is
  N(0,1) plus GAMMA times the unit vector of LM-head row t*_u, which makes t*_u the target's
  argmax with overwhelming probability.  A child carries its parent's planted token with the
  configured match probability (at most one sibling does), else a uniform random token distinct
  from its siblings and from t*_u.  With `target_argmax` given (a function of the hidden rows
  and the head that returns each row's argmax, supplied by the caller), the hidden states are
  plain N(0,1) and t*_u is that function's answer instead: the natural recipe, whose top-1 /
  top-2 margins are those of N(0, 1.43) logits over the whole vocabulary.
* T>0: target logits come out N(0,2) by drawing W ~ N(0, 2/sqrt(hidden)); draft distributions
  are softmax of N(0,2) logits and each draft token is sampled from its parent's draft
  distribution, independently for siblings (chains and branching trees alike).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np
import torch

# Strength of the planted-argmax direction in the T=0 hidden states (in units of the logit std).
GAMMA = 10.0

# Tags that keep every named random stream independent of the others and of tensor sizes.
_TAGS = {
    "tree": 1, "tokens": 2, "plant": 3, "q": 4, "k_tree": 5, "v_tree": 6, "k_cache": 7,
    "v_cache": 8, "hidden": 9, "w_lm": 10, "kv_len": 11, "draft_logits": 12, "draft_pick": 13,
    "pages": 14, "lr_u": 15, "lr_d": 16, "lr_noise": 17, "lr_hidden": 18,
}

CONFIGS: dict[str, dict] = {
    # 1 request, 1 layer, 8/2 heads, hidden 1024, vocab 4096, KV 512, 16-node tree (depth<=6,
    # branching<=4), match 0.7, greedy.
    "tiny": dict(B=1, hq=8, hkv=2, head_dim=128, hidden=1024, vocab=4096, kv_len=(512, 512),
                 n_nodes=16, depth=6, depth_min=6, branch=4, width=None, match=0.7,
                 temperature=0.0, w_sigma=0.02),
    # 27B-class dense shape, 1 request, KV 4096, 64-node tree (depth 8, width<=16), match 0.75.
    "dense27b_b1": dict(B=1, hq=40, hkv=8, head_dim=128, hidden=5120, vocab=151936,
                        kv_len=(4096, 4096), n_nodes=64, depth=8, depth_min=8, branch=None,
                        width=16, match=0.75, temperature=0.0, w_sigma=0.02),
    # long context, 1 request, 16-node tree of depth 6.
    "long32k": dict(B=1, hq=40, hkv=8, head_dim=128, hidden=5120, vocab=151936,
                    kv_len=(32768, 32768), n_nodes=16, depth=6, depth_min=6, branch=4,
                    width=None, match=0.75, temperature=0.0, w_sigma=0.02),
    "long128k": dict(B=1, hq=40, hkv=8, head_dim=128, hidden=5120, vocab=151936,
                     kv_len=(131072, 131072), n_nodes=16, depth=6, depth_min=6, branch=4,
                     width=None, match=0.75, temperature=0.0, w_sigma=0.02),
    # 64 concurrent requests, KV ~ U[1024, 8192], independent random 16-node trees.
    "batch64": dict(B=64, hq=40, hkv=8, head_dim=128, hidden=5120, vocab=151936,
                    kv_len=(1024, 8192), n_nodes=16, depth=6, depth_min=2, branch=4,
                    width=None, match=0.7, temperature=0.0, w_sigma=0.02),
    # 512 concurrent requests, KV ~ U[512, 4096], 4-node chains, stochastic acceptance at T=1.
    "conc512": dict(B=512, hq=40, hkv=8, head_dim=128, hidden=5120, vocab=151936,
                    kv_len=(512, 4096), n_nodes=4, depth=3, depth_min=3, branch=1, width=None,
                    match=None, temperature=1.0, w_sigma=None, draft_sigma=2.0),
    # 64 requests, KV ~ U[1024, 8192], branching 16-node trees (<= 4 children per node),
    # stochastic acceptance at T=1 with siblings drafted independently.
    "tree64_t1": dict(B=64, hq=40, hkv=8, head_dim=128, hidden=5120, vocab=151936,
                      kv_len=(1024, 8192), n_nodes=16, depth=6, depth_min=2, branch=4,
                      width=None, match=None, temperature=1.0, w_sigma=None, draft_sigma=2.0),
}
CONFIG_INDEX = {"tiny": 0, "dense27b_b1": 1, "long32k": 2, "long128k": 2, "batch64": 3,
                "conc512": 4, "tree64_t1": 5}


def config_seed(name: str) -> int:
    return 0xE7EE0000 + CONFIG_INDEX.get(name, 0)


@dataclass
class Workload:
    name: str
    cfg: dict
    seed: int
    step: int
    B: int
    hq: int
    hkv: int
    head_dim: int
    hidden_dim: int
    vocab: int
    temperature: float
    # tree / batch description (host int arrays)
    cu_nodes: np.ndarray        # int32 [B+1]
    parent: np.ndarray          # int32 [n_total], local indices, parent[root] = -1
    tokens: np.ndarray          # int32 [n_total]
    kv_len: np.ndarray          # int32 [B]
    slot_base: np.ndarray       # int64 [B]
    slot_cap: np.ndarray        # int32 [B]
    planted: np.ndarray         # int32 [n_total] planted target token per node (-1 if none)
    # tensors (torch CPU; bf16 unless stated)
    q: torch.Tensor             # [n_total, hq, D]
    k_tree: torch.Tensor        # [n_total, hkv, D]
    v_tree: torch.Tensor        # [n_total, hkv, D]
    k_cache: torch.Tensor       # [slots, hkv, D]
    v_cache: torch.Tensor       # [slots, hkv, D]
    hidden: torch.Tensor        # [n_total, H]
    w_lm: torch.Tensor          # [V, H]
    q_draft: torch.Tensor | None = None   # fp32 [n_total, V] (T>0 only)
    extra: dict = field(default_factory=dict)

    @property
    def n_total(self) -> int:
        return int(self.cu_nodes[-1])

    @property
    def n_max(self) -> int:
        return int(np.max(np.diff(self.cu_nodes)))

    @property
    def kv_len_max(self) -> int:
        return int(np.max(self.kv_len))

    @property
    def slots(self) -> int:
        return int(self.k_cache.shape[0])

    def nodes(self, r: int) -> int:
        return int(self.cu_nodes[r + 1] - self.cu_nodes[r])


def _rng(seed: int, tag: str, *ids: int) -> np.random.Generator:
    return np.random.default_rng([seed, _TAGS[tag], *ids])


def _threads() -> int:
    try:
        return max(1, min(32, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover
        return max(1, min(32, os.cpu_count() or 1))


def normal_f32(n: int, sigma: float, seed: int, tag: str) -> np.ndarray:
    """n fp32 samples of N(0, sigma), filled in parallel from independent chunk streams.

    The chunking is fixed (1 Mi samples per chunk, each chunk its own seeded stream), so the
    values depend only on (seed, tag, n), not on the thread count.
    """
    out = np.empty(n, dtype=np.float32)
    chunk = 1 << 20
    nchunks = (n + chunk - 1) // chunk

    def fill(c: int) -> None:
        lo, hi = c * chunk, min(n, (c + 1) * chunk)
        g = np.random.default_rng([seed, _TAGS[tag], 0xC0FFEE, c])
        g.standard_normal(out=out[lo:hi], dtype=np.float32)
        if sigma != 1.0:
            out[lo:hi] *= np.float32(sigma)

    if nchunks <= 1:
        fill(0) if n else None
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(nchunks)))
    return out


def normal_bf16(shape, sigma: float, seed: int, tag: str) -> torch.Tensor:
    n = int(np.prod(shape))
    f = normal_f32(n, sigma, seed, tag)
    # torch's CPU cast rounds to nearest-even
    return torch.from_numpy(f).to(torch.bfloat16).reshape(*shape)


def make_tree(n: int, depth: int, branch, width, rng: np.random.Generator) -> np.ndarray:
    """Random tree with n nodes (root included), BFS-ordered so that parent[i] < i."""
    if n < 1:
        raise ValueError("a tree has at least its root")
    depth = min(depth, n - 1)
    par = [-1]
    dep = [0]
    nchild = [0]
    level = {0: 1}
    for d in range(1, depth + 1):          # the spine
        par.append(d - 1)
        dep.append(d)
        nchild.append(0)
        nchild[d - 1] += 1
        level[d] = level.get(d, 0) + 1
    while len(par) < n:
        elig = [u for u in range(len(par))
                if dep[u] < depth
                and (branch is None or nchild[u] < branch)
                and (width is None or level.get(dep[u] + 1, 0) < width)]
        if not elig:
            raise ValueError("tree caps leave no room for another node")
        u = int(elig[rng.integers(len(elig))])
        par.append(u)
        dep.append(dep[u] + 1)
        nchild.append(0)
        nchild[u] += 1
        level[dep[u] + 1] = level.get(dep[u] + 1, 0) + 1
    # relabel in BFS order (children in insertion order)
    children = [[] for _ in range(n)]
    for i in range(1, n):
        children[par[i]].append(i)
    order = [0]
    head = 0
    while head < len(order):
        order.extend(children[order[head]])
        head += 1
    new_of = {old: new for new, old in enumerate(order)}
    out = np.full(n, -1, dtype=np.int32)
    for old in range(1, n):
        out[new_of[old]] = new_of[par[old]]
    return out


def _draft_tokens_greedy(parent: np.ndarray, planted: np.ndarray, vocab: int, match: float,
                         rng: np.random.Generator) -> np.ndarray:
    n = len(parent)
    tok = np.empty(n, dtype=np.int32)
    tok[0] = rng.integers(vocab)
    children = [[] for _ in range(n)]
    for i in range(1, n):
        children[parent[i]].append(i)
    for u in range(n):
        target = int(planted[u])
        matched = False
        used = {target}
        for c in children[u]:
            coin = rng.random() < match
            if coin and not matched:
                tok[c] = target
                matched = True
                continue
            while True:
                t = int(rng.integers(vocab))
                if t not in used:
                    break
            used.add(t)
            tok[c] = t
    return tok


def generate(name: str, *, seed: int | None = None, step: int = 0, target_argmax=None,
             **overrides) -> Workload:
    """Build the named workload (overrides replace config fields, e.g. vocab=4224).

    target_argmax (T = 0 only): callable(hidden bf16 [n, H], w_lm bf16 [V, H]) -> int array [n]
    of each row's argmax; when given, hidden states are unplanted N(0, 1) and the drafts follow
    the returned argmaxes (see the module notes)."""
    cfg = dict(CONFIGS[name])
    cfg.update(overrides)
    seed = config_seed(name) if seed is None else int(seed)
    B, hq, hkv, D = cfg["B"], cfg["hq"], cfg["hkv"], cfg["head_dim"]
    H, V = cfg["hidden"], cfg["vocab"]
    T = float(cfg["temperature"])

    # --- per-request trees, lengths and tokens
    if isinstance(cfg["kv_len"], list):            # explicit per-request lengths
        kv_len = np.asarray(cfg["kv_len"], dtype=np.int32)
        assert len(kv_len) == B
    else:
        lo, hi = cfg["kv_len"]
        kv_len = _rng(seed, "kv_len").integers(lo, hi + 1, size=B).astype(np.int32) \
            if hi > lo else np.full(B, lo, dtype=np.int32)
    n_nodes = cfg["n_nodes"]
    n_nodes = list(n_nodes) if isinstance(n_nodes, (list, tuple)) else [n_nodes] * B
    assert len(n_nodes) == B
    parents, sizes = [], []
    for r in range(B):
        g = _rng(seed, "tree", r)
        dmin = cfg.get("depth_min", cfg["depth"])
        d = int(g.integers(dmin, cfg["depth"] + 1)) if dmin < cfg["depth"] else cfg["depth"]
        p = make_tree(int(n_nodes[r]), d, cfg["branch"], cfg["width"], g)
        parents.append(p)
        sizes.append(len(p))
    cu = np.zeros(B + 1, dtype=np.int32)
    cu[1:] = np.cumsum(sizes)
    ntot = int(cu[-1])
    parent = np.concatenate(parents).astype(np.int32)

    slot_cap = (kv_len + 64).astype(np.int32)
    slot_base = np.zeros(B, dtype=np.int64)
    slot_base[1:] = np.cumsum(slot_cap.astype(np.int64))[:-1]
    slots = int(slot_base[-1] + slot_cap[-1])

    # --- dense tensors
    q = normal_bf16((ntot, hq, D), 1.0, seed, "q")
    k_tree = normal_bf16((ntot, hkv, D), 1.0, seed, "k_tree")
    v_tree = normal_bf16((ntot, hkv, D), 1.0, seed, "v_tree")
    k_cache = normal_bf16((slots, hkv, D), 1.0, seed, "k_cache")
    v_cache = normal_bf16((slots, hkv, D), 1.0, seed, "v_cache")

    q_draft = None
    planted = np.full(ntot, -1, dtype=np.int32)
    if T == 0.0:
        w_lm = normal_bf16((V, H), cfg["w_sigma"], seed, "w_lm")
        h = normal_f32(ntot * H, 1.0, seed, "hidden").reshape(ntot, H)
        tokens = np.empty(ntot, dtype=np.int32)
        if target_argmax is not None:
            hidden = torch.from_numpy(h).to(torch.bfloat16)
            planted[:] = np.asarray(target_argmax(hidden, w_lm), dtype=np.int32)
        for r in range(B):
            a, b = int(cu[r]), int(cu[r + 1])
            if target_argmax is None:
                planted[a:b] = _rng(seed, "plant", r).integers(V, size=b - a)
            tokens[a:b] = _draft_tokens_greedy(parent[a:b], planted[a:b], V, cfg["match"],
                                               _rng(seed, "tokens", r))
        if target_argmax is None:
            rows = w_lm[torch.from_numpy(planted.astype(np.int64))].float().numpy()
            rows /= np.linalg.norm(rows, axis=1, keepdims=True)
            h += np.float32(GAMMA) * rows
            hidden = torch.from_numpy(h).to(torch.bfloat16)
    else:
        w_lm = normal_bf16((V, H), 2.0 / np.sqrt(H), seed, "w_lm")
        hidden = normal_bf16((ntot, H), 1.0, seed, "hidden")
        d = normal_f32(ntot * V, cfg.get("draft_sigma", 2.0), seed, "draft_logits")
        d = d.reshape(ntot, V)
        q_np = np.empty((ntot, V), dtype=np.float32)
        tokens = np.empty(ntot, dtype=np.int32)
        pick = _rng(seed, "draft_pick")
        for i in range(ntot):
            row = d[i].astype(np.float64)
            e = np.exp(row - row.max())
            q_np[i] = (e / e.sum()).astype(np.float32)
        u = pick.random(ntot)
        for r in range(B):
            a, b = int(cu[r]), int(cu[r + 1])
            tokens[a] = int(pick.integers(V))
            for i in range(a + 1, b):
                pr = a + int(parent[i])
                c = np.cumsum(q_np[pr].astype(np.float64))
                tokens[i] = int(min(V - 1, np.searchsorted(c, u[i] * c[-1], side="right")))
        q_draft = torch.from_numpy(q_np)

    return Workload(name=name, cfg=cfg, seed=seed, step=step, B=B, hq=hq, hkv=hkv, head_dim=D,
                    hidden_dim=H, vocab=V, temperature=T, cu_nodes=cu, parent=parent,
                    tokens=tokens, kv_len=kv_len, slot_base=slot_base, slot_cap=slot_cap,
                    planted=planted, q=q, k_tree=k_tree, v_tree=v_tree, k_cache=k_cache,
                    v_cache=v_cache, hidden=hidden, w_lm=w_lm, q_draft=q_draft)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Zero-copy uint16 view of a contiguous CPU bf16 tensor."""
    assert t.dtype == torch.bfloat16 and t.is_contiguous()
    return t.view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------------------- paged layout
@dataclass
class PagedCache:
    """A workload's cache laid out in pages of a shared pool (the input of the paged calls)."""
    page_size: int
    max_pages: int
    num_pages: int
    block_table: np.ndarray          # int32 [B, max_pages], -1 where no page is mapped
    k_pool: torch.Tensor             # bf16 [num_pages * page_size, hkv, d]
    v_pool: torch.Tensor
    slot_cap: np.ndarray             # int32 [B]: mapped pages x page_size


def paged(wl: "Workload", page_size: int, spare_pages: int = 3, seed: int = 0) -> PagedCache:
    """Lays the workload's per-request caches out in page_size-token pages at random distinct
    pool pages (plus unmapped spare pages): logical position t of request r goes to pool slot
    block_table[r, t // page_size] * page_size + t % page_size.  Each request maps
    ceil(slot_cap[r] / page_size) pages, so its capacity is that many pages."""
    g = _rng(wl.seed, "pages", seed)
    P = int(page_size)
    npg = [(int(c) + P - 1) // P for c in wl.slot_cap]
    total = sum(npg) + spare_pages
    perm = g.permutation(total).astype(np.int32)
    maxp = max(npg) if npg else 1
    bt = np.full((wl.B, maxp), -1, dtype=np.int32)
    kp = torch.zeros((total * P,) + tuple(wl.k_cache.shape[1:]), dtype=torch.bfloat16)
    vp = torch.zeros_like(kp)
    nxt = 0
    for r in range(wl.B):
        base, cap = int(wl.slot_base[r]), int(wl.slot_cap[r])
        for j in range(npg[r]):
            page = int(perm[nxt])
            nxt += 1
            bt[r, j] = page
            lo, hi = j * P, min(cap, (j + 1) * P)
            kp[page * P:page * P + hi - lo] = wl.k_cache[base + lo:base + hi]
            vp[page * P:page * P + hi - lo] = wl.v_cache[base + lo:base + hi]
    return PagedCache(page_size=P, max_pages=maxp, num_pages=total, block_table=bt, k_pool=kp,
                      v_pool=vp, slot_cap=np.array([n * P for n in npg], dtype=np.int32))


# ----------------------------------------------------------------- low-rank candidate head
LOWRANK = {
    # the draft head's shape at the 27B-class vocabulary: 64 tree nodes per call
    "lowrank_r512": dict(M=64, H=5120, V=151936, r=512, k=16),
    "lowrank_r128": dict(M=64, H=5120, V=151936, r=128, k=16),
    "lowrank_tiny": dict(M=9, H=256, V=4096 + 77, r=64, k=8),
}


@dataclass
class LowRankWorkload:
    name: str
    M: int
    H: int
    V: int
    r: int
    k: int
    hidden: torch.Tensor     # bf16 [M, H]
    D: torch.Tensor          # bf16 [r, H]
    U: torch.Tensor          # bf16 [V, r]
    W: torch.Tensor          # bf16 [V, H]


def lowrank(name: str, **over) -> LowRankWorkload:
    """Factors and head of a low-rank candidate screen.  U, D ~ N(0, s) with s^4 r = 0.02^2, so
    U D has the full head's N(0, 0.02) scale; the exact head is W = U D + N(0, 0.005) (a head
    that the factors approximate but do not equal); hidden rows N(0, 1)."""
    cfg = dict(LOWRANK[name])
    cfg.update(over)
    M, H, V, r, k = cfg["M"], cfg["H"], cfg["V"], cfg["r"], cfg["k"]
    seed = 0xE7EE0100 + sum(map(ord, name))
    s = (0.02 ** 2 / r) ** 0.25
    Uf = normal_f32(V * r, s, seed, "lr_u").reshape(V, r)
    Df = normal_f32(r * H, s, seed, "lr_d").reshape(r, H)
    Ub = torch.from_numpy(Uf).to(torch.bfloat16)
    Db = torch.from_numpy(Df).to(torch.bfloat16)
    Wf = torch.from_numpy(normal_f32(V * H, 0.005, seed, "lr_noise").reshape(V, H))
    Wf += Ub.float() @ Db.float()
    hidden = torch.from_numpy(normal_f32(M * H, 1.0, seed, "lr_hidden").reshape(M, H))
    return LowRankWorkload(name=name, M=M, H=H, V=V, r=r, k=k,
                           hidden=hidden.to(torch.bfloat16), D=Db, U=Ub,
                           W=Wf.to(torch.bfloat16))
