"""The CUDA samplers against the target distribution itself (chi-square through the C ABI).

Verification at T > 0 must leave the target's output distribution unchanged: the token emitted
at every position follows the target's softmax, whatever the draft proposed ("Eagle-4 Released:
Outpaces DFlash2 and DSpark ...", section "Technical Background"; "EAGLE-4 官方推理代码发布 ...",
section on sizing the speculative tree by measured cost, which keeps the output distribution).
These tests run the GPU's accept tests and bonus draws on 10^6 trials and compare the emitted
tokens with p, independently of the fp64 oracle's own sampler: the expected distribution is
the softmax of the fp64 logits of the same bf16 inputs, and the acceptance rates are the closed
forms of speculative sampling.

Each trial is one request of a large batch; trials differ by request index and by the call's
step, which key the library's uniforms, and by the draft tokens, drawn here from q.
"""
import numpy as np
import pytest
import torch
from scipy import stats

import draft_tree_verification_masked_b200 as et

import oracle

pytestmark = pytest.mark.gpu

V, H, R = 256, 64, 4096          # vocabulary, hidden size, requests (trials) per call
CALLS = 250                      # 1,024,000 trials


def _softmax(x):
    e = np.exp(x - x.max())
    return e / e.sum()


def _chisq_p(samples, probs, min_expected=5.0):
    """Chi-square p-value of the samples against probs, rare ids pooled into one bin."""
    counts = np.bincount(samples, minlength=len(probs)).astype(np.float64)
    exp = probs * len(samples)
    assert counts[probs == 0].sum() == 0
    big = exp >= min_expected
    c = np.append(counts[big], counts[~big].sum())
    e = np.append(exp[big], exp[~big].sum())
    keep = e > 0
    return stats.chisquare(c[keep], e[keep]).pvalue


class _Setup:
    """Head, hidden rows and draft rows of a V-token toy target, and a batch of R requests of
    n nodes each with parent array `par` (the same shape for every request)."""

    def __init__(self, par, seed, q_scale=None, full=False):
        g = np.random.default_rng(seed)
        self.n = len(par)
        hid = torch.from_numpy(g.normal(0, 1, size=(self.n, H)).astype(np.float32)).bfloat16()
        w = torch.from_numpy(g.normal(0, 1.5 / np.sqrt(H), size=(V, H)).astype(np.float32))
        self.w = w.bfloat16()
        z = oracle.logits(hid, self.w, np.arange(self.n, dtype=np.int32))
        self.p = np.stack([_softmax(zr) for zr in z])              # fp64 target rows
        if q_scale is None:
            self.q = np.stack([_softmax(g.normal(0, 1.5, size=V)) for _ in range(self.n)])
        else:                                                      # q = q_scale * p
            self.q = q_scale * self.p
        self.q32 = self.q.astype(np.float32)
        self.g = g
        dev = torch.device("cuda")
        i32 = dict(dtype=torch.int32, device=dev)
        self.cu = torch.arange(0, R * self.n + 1, self.n, **i32)
        self.parent = torch.tensor(np.tile(np.asarray(par, np.int32), R), **i32)
        self.tokens = torch.zeros(R * self.n, **i32)
        self.kv_len = torch.zeros(R, **i32)
        self.slot_cap = torch.full((R,), 64, **i32)
        self.slot_base = torch.arange(R, dtype=torch.int64, device=dev) * 64
        self.batch = et.make_batch(self.cu, self.parent, self.tokens, self.kv_len,
                                   self.slot_base, self.slot_cap, self.n, 0)
        self.hidden = hid.repeat(R, 1).to(dev)
        self.w_lm = self.w.to(dev)
        self.q_draft = torch.from_numpy(np.tile(self.q32, (R, 1))).to(dev)
        self.ws = torch.zeros(et.etree_workspace_size(self.batch, 0, 0, 128, H, V),
                              dtype=torch.uint8, device=dev)
        et.etree_workspace_init(self.ws)
        self.accept_len = torch.empty(R, **i32)
        self.path = torch.empty(R, 64, **i32)
        self.out = torch.empty(R, 65, **i32)
        self.node_argmax = torch.empty(R * self.n, **i32)
        self.node_gap = torch.empty(R * self.n, dtype=torch.float32, device=dev)
        # a row per branching node (the root), or with `full` a row per node: the draw then
        # reads the stored stop rows instead of a second pass over the head
        self.zbuf = torch.empty(R * (self.n if full else 1), V, dtype=torch.float32, device=dev)

    def draft(self, parent_rows):
        """Draft tokens for the given parent rows of every request, each drawn from that row's q
        (float32 values, as the library reads them)."""
        cq = np.cumsum(self.q32.astype(np.float64), axis=1)
        toks = np.empty((R, len(parent_rows)), dtype=np.int32)
        for j, u in enumerate(parent_rows):
            toks[:, j] = np.minimum(V - 1, np.searchsorted(cq[u], self.g.random(R) * cq[u, -1],
                                                           side="right"))
        return toks

    def run(self, tokens, step, tree=False):
        self.tokens.copy_(torch.from_numpy(tokens.reshape(-1)))
        if tree:
            et.etree_lmhead_accept_tree(self.batch, self.hidden, self.w_lm, 1.0, self.q_draft,
                                        0xE7EE0900, step, self.accept_len, self.path, self.out,
                                        self.zbuf, self.ws)
        else:
            et.etree_lmhead_accept(self.batch, self.hidden, self.w_lm, 1.0, self.q_draft,
                                   0xE7EE0900, step, self.accept_len, self.path, self.out,
                                   self.node_argmax, self.node_gap, self.ws)
        assert et.etree_device_status(self.ws) == (0, 0)
        return (self.accept_len.cpu().numpy(), self.path.cpu().numpy(), self.out.cpu().numpy())


@pytest.mark.parametrize("mode", ["chain", "materialised"])
def test_chain_sampler_emits_the_target_distribution(mode):
    """2-node chains: the first emitted token (the accepted draft, or the residual draw after a
    rejection) follows p_root; the draft is accepted with probability sum min(p, q); after an
    acceptance the bonus follows p of the child.  `materialised`: the same through the tree entry
    with every row's logits kept, whose draw reads the stored rows."""
    full = mode == "materialised"
    s = _Setup([-1, 0], seed=91, full=full)
    first, second, acc = [], [], []
    for step in range(CALLS):
        tok = np.zeros((R, 2), dtype=np.int32)
        tok[:, 1] = s.draft([0])[:, 0]
        a, path, out = s.run(tok, step, tree=full)
        assert set(np.unique(a)) <= {0, 1}
        first.append(out[:, 0])
        second.append(out[a == 1, 1])
        acc.append(a)
    first, second, acc = map(np.concatenate, (first, second, acc))
    assert _chisq_p(first, s.p[0]) > 1e-4
    want = np.minimum(s.p[0], s.q[0]).sum()
    assert abs(acc.mean() - want) < 5 * np.sqrt(want * (1 - want) / len(acc))
    assert _chisq_p(second, s.p[1]) > 1e-4


@pytest.mark.parametrize("full", [False, True])
def test_tree_sampler_emits_the_target_distribution_and_sibling_rates(full):
    """A root with three children drafted independently from q_root: the first emitted token
    follows p_root; child 1 is accepted with A1 = sum min(p, q); after its rejection the target
    is r1 = max(0, p - q) / (1 - A1) and child 2 is accepted with sum min(q, r1); after both
    rejections r2 = max(0, p - c2 q) / N(c2) with c2 = 2 - A1, and child 3 with sum min(q, r2).
    With `full`, every row's logits are kept and the draw reads them."""
    s = _Setup([-1, 0, 0, 0], seed=92, full=full)
    first, which = [], []
    for step in range(CALLS):
        tok = np.zeros((R, 4), dtype=np.int32)
        tok[:, 1:] = s.draft([0, 0, 0])
        a, path, out = s.run(tok, step, tree=True)
        first.append(out[:, 0])
        which.append(np.where(a >= 1, path[:, 1], 0))
    first, which = np.concatenate(first), np.concatenate(which)
    n = len(first)
    assert _chisq_p(first, s.p[0]) > 1e-4
    p, q = s.p[0], s.q32[0].astype(np.float64)
    A1 = np.minimum(p, q).sum()
    r1 = np.maximum(0.0, p - q) / (1.0 - A1)
    A2 = np.minimum(q, r1).sum()
    c2 = 2.0 - A1
    N2 = np.maximum(0.0, p - c2 * q).sum()
    r2 = np.maximum(0.0, p - c2 * q) / N2
    A3 = np.minimum(q, r2).sum()
    for k, want in ((1, A1), (2, (1 - A1) * A2), (3, (1 - A1) * (1 - A2) * A3)):
        got = (which == k).mean()
        assert abs(got - want) < 5 * np.sqrt(want * (1 - want) / n), (k, got, want)


@pytest.mark.parametrize("tree,full", [(False, False), (True, False), (True, True)])
def test_empty_residual_bonus_is_drawn_from_the_target(tree, full):
    """q = 2p (an over-confident draft): every residual max(0, p - q) is empty, so each rejection
    (probability 1/2) is answered by a draw from p itself; together with the accepted drafts
    (x ~ q / 2 = p) the first emitted token follows p, and so does the bonus alone."""
    par = [-1, 0, 0] if tree else [-1, 0]
    s = _Setup(par, seed=93, q_scale=2.0, full=full)
    first, rej = [], []
    calls = CALLS // 5
    for step in range(calls):
        tok = np.zeros((R, len(par)), dtype=np.int32)
        cp = np.cumsum(s.p[0])
        for j in range(1, len(par)):
            tok[:, j] = np.minimum(V - 1, np.searchsorted(cp, s.g.random(R) * cp[-1],
                                                          side="right"))
        a, path, out = s.run(tok, step, tree=tree)
        first.append(out[:, 0])
        rej.append(a == 0)
    first, rej = np.concatenate(first), np.concatenate(rej)
    want = 0.5          # a tree stops at its first rejection: the residual has no weight left
    assert abs(rej.mean() - want) < 5 * np.sqrt(want * (1 - want) / len(rej))
    assert _chisq_p(first[rej], s.p[0]) > 1e-4
    assert _chisq_p(first, s.p[0]) > 1e-4
