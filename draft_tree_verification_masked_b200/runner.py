"""Device-side driver of one verification step over a workload (marshalling only).

Uploads a :class:`~draft_tree_verification_masked_b200.workload.Workload` to the GPU, allocates
the outputs and the workspace with PyTorch, and calls the three C-ABI entry points in order:
tree attention (one layer), LM head + acceptance, KV compaction.
"""
from __future__ import annotations

import torch

import numpy as np

from . import (etree_device_status, etree_kv_compact, etree_kv_compact_paged,
               etree_lmhead_accept, etree_lmhead_accept_timed, etree_lmhead_accept_tree,
               etree_verify_attn,
               etree_verify_attn_paged, etree_workspace_init, etree_workspace_size, make_batch)


def branching_nodes(wl) -> int:
    """Number of tree nodes with two or more children."""
    cnt = np.zeros(wl.n_total, dtype=np.int64)
    for r in range(wl.B):
        a0, a1 = int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])
        par = np.asarray(wl.parent[a0 + 1:a1], dtype=np.int64)
        np.add.at(cnt, a0 + par, 1)
    return int((cnt >= 2).sum())


class Packed:
    """Tensors laid out back to back, each at a 256-byte boundary, in one device byte buffer."""

    def __init__(self, specs, device):
        self.slots = {}
        off = 0
        for name, shape, dtype in specs:
            nbytes = int(np.prod(shape, dtype=np.int64)) * torch.empty((), dtype=dtype).element_size()
            self.slots[name] = (off, tuple(shape), dtype, nbytes)
            off = (off + nbytes + 255) // 256 * 256
        self.buf = torch.zeros(max(off, 256), dtype=torch.uint8, device=device)

    def view(self, name):
        off, shape, dtype, nbytes = self.slots[name]
        return self.buf[off:off + nbytes].view(dtype).view(shape)

    def offset(self, name) -> int:
        """Byte offset of a tensor in the buffer (tensors after it follow contiguously)."""
        return self.slots[name][0]


class DeviceStep:
    """tree: None picks the branching-tree sampler (etree_lmhead_accept_tree) when T > 0 and a
    node has two or more children; zbuf_rows overrides the size of its logit buffer.
    page_size: lay the caches out in pages of that many tokens at shuffled pool pages and use
    the paged attention and compaction calls (the pools replace k_cache / v_cache).
    kv_len_max: the batch's host-side bound on kv_len (default: the largest kv_len); a looser
    bound is valid and sizes the attention grid for it.
    materialize (T > 0): use the tree entry point with a logit buffer of n_total rows, so that the
    bonus draw reads the stop rows' stored logits instead of making a second pass over the head."""

    def __init__(self, wl, device: str = "cuda", n_layers: int = 1, tree=None, zbuf_rows=None,
                 page_size=None, kv_len_max=None, materialize: bool = False):
        self.wl = wl
        self.device = device
        dev = torch.device(device)
        i32 = torch.int32

        def up(x, dtype=None):
            t = torch.as_tensor(x) if not isinstance(x, torch.Tensor) else x
            if dtype is not None:
                t = t.to(dtype)
            return t.contiguous().to(dev)

        self.paged = None
        if page_size:
            from .workload import paged
            self.paged = paged(wl, int(page_size))
        # The per-step inputs live back to back in one device buffer (`inputs.buf`), and the
        # accept results in another (`outputs.buf`), so that a serving loop moves each direction
        # in a single copy.  The attention's inputs come first and the LM head's (hidden states,
        # draft probabilities) last, from byte `inputs.offset("hidden")` on, so the second part
        # can be copied while the attention runs.  The caches and the LM-head weight stay
        # resident on their own.
        srcs = [("cu_nodes", wl.cu_nodes, i32), ("parent", wl.parent, i32),
                ("tokens", wl.tokens, i32), ("kv_len", wl.kv_len, i32),
                ("slot_base", wl.slot_base, torch.int64),
                ("slot_cap", self.paged.slot_cap if self.paged else wl.slot_cap, i32)]
        if self.paged:
            srcs.append(("block_table", self.paged.block_table, i32))
        srcs += [("q", wl.q, None), ("k_tree", wl.k_tree, None), ("v_tree", wl.v_tree, None),
                 ("hidden", wl.hidden, None)]
        if wl.q_draft is not None:
            srcs.append(("q_draft", wl.q_draft, None))
        host = {}
        for name, x, dtype in srcs:
            t = torch.as_tensor(x) if not isinstance(x, torch.Tensor) else x
            host[name] = (t.to(dtype) if dtype is not None else t).contiguous()
        self.inputs = Packed([(k, tuple(t.shape), t.dtype) for k, t in host.items()], dev)
        for name, t in host.items():
            v = self.inputs.view(name)
            v.copy_(t)
            setattr(self, name, v)
        self.batch = make_batch(self.cu_nodes, self.parent, self.tokens, self.kv_len,
                                self.slot_base, self.slot_cap, wl.n_max,
                                wl.kv_len_max if kv_len_max is None else int(kv_len_max))
        self.k_cache = up(self.paged.k_pool if self.paged else wl.k_cache)
        self.v_cache = up(self.paged.v_pool if self.paged else wl.v_cache)
        self.w_lm = up(wl.w_lm)
        self.q_draft = up(wl.q_draft) if wl.q_draft is not None else None
        ntot, B = wl.n_total, wl.B
        self.out = torch.empty(ntot, wl.hq, wl.head_dim, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(ntot, wl.hq, dtype=torch.float32, device=dev)
        self.outputs = Packed([("accept_len", (B,), i32), ("path", (B, 64), i32),
                               ("out_tokens", (B, 65), i32)], dev)
        self.accept_len = self.outputs.view("accept_len")
        self.path = self.outputs.view("path")
        self.out_tokens = self.outputs.view("out_tokens")
        self.node_argmax = torch.empty(ntot, dtype=i32, device=dev)
        self.node_gap = torch.empty(ntot, dtype=torch.float32, device=dev)
        self.kv_len_out = torch.empty(B, dtype=i32, device=dev)
        self.n_layers = n_layers
        if n_layers == 1:
            self.kt_layers, self.vt_layers = self.k_tree, self.v_tree
            self.kc_layers, self.vc_layers = self.k_cache, self.v_cache
        else:
            # stacked per-layer copies; layer 0 holds the workload's tensors
            self.kt_layers = self.k_tree.unsqueeze(0).repeat(n_layers, 1, 1, 1)
            self.vt_layers = self.v_tree.unsqueeze(0).repeat(n_layers, 1, 1, 1)
            self.kc_layers = torch.zeros((n_layers,) + tuple(self.k_cache.shape),
                                         dtype=torch.bfloat16, device=dev)
            self.vc_layers = torch.zeros_like(self.kc_layers)
        self.tree_layer_stride = self.k_tree.numel()
        self.cache_layer_stride = self.k_cache.numel()
        size = etree_workspace_size(self.batch, wl.hq, wl.hkv, wl.head_dim, wl.hidden_dim,
                                    wl.vocab)
        self.ws = torch.zeros(max(size, 256), dtype=torch.uint8, device=dev)
        etree_workspace_init(self.ws)
        self.scale = 1.0 / float(wl.head_dim) ** 0.5
        nbr = branching_nodes(wl)
        self.materialize = bool(materialize) and wl.temperature > 0
        if self.materialize:
            tree, zbuf_rows = True, wl.n_total
        self.tree = (wl.temperature > 0 and nbr > 0) if tree is None else bool(tree)
        rows = nbr if zbuf_rows is None else int(zbuf_rows)
        self.zbuf = (torch.empty(rows, wl.vocab, dtype=torch.float32, device=dev)
                     if self.tree and rows > 0 else None)

    # --- the three calls
    def attn(self, stream=None):
        if self.paged:
            etree_verify_attn_paged(self.batch, self.block_table, self.paged.page_size, self.q,
                                    self.k_tree, self.v_tree, self.k_cache, self.v_cache,
                                    self.scale, self.out, self.lse, self.ws, stream)
            return
        etree_verify_attn(self.batch, self.q, self.k_tree, self.v_tree, self.k_cache,
                          self.v_cache, self.scale, self.out, self.lse, self.ws, stream)

    def lmhead(self, stream=None):
        if self.tree:
            etree_lmhead_accept_tree(self.batch, self.hidden, self.w_lm, self.wl.temperature,
                                     self.q_draft, self.wl.seed, self.wl.step, self.accept_len,
                                     self.path, self.out_tokens, self.zbuf, self.ws, stream)
            return
        etree_lmhead_accept(self.batch, self.hidden, self.w_lm, self.wl.temperature,
                            self.q_draft, self.wl.seed, self.wl.step, self.accept_len, self.path,
                            self.out_tokens, self.node_argmax, self.node_gap, self.ws, stream)

    def lmhead_marked(self, marks, stream=None):
        """The LM-head call with its phase marks (see etree_lmhead_accept_timed)."""
        etree_lmhead_accept_timed(self.batch, self.hidden, self.w_lm, self.wl.temperature,
                                  self.q_draft, self.wl.seed, self.wl.step, self.accept_len,
                                  self.path, self.out_tokens, self.node_argmax, self.node_gap,
                                  self.zbuf, self.tree, marks, self.ws, stream)

    def compact(self, stream=None):
        if self.paged:
            etree_kv_compact_paged(self.batch, self.block_table, self.paged.page_size,
                                   self.accept_len, self.path, self.kt_layers, self.vt_layers,
                                   self.kc_layers, self.vc_layers, self.paged.num_pages,
                                   self.n_layers, self.tree_layer_stride,
                                   self.cache_layer_stride, self.kv_len_out, self.ws, stream)
            return
        etree_kv_compact(self.batch, self.accept_len, self.path, self.kt_layers, self.vt_layers,
                         self.kc_layers, self.vc_layers, self.n_layers, self.tree_layer_stride,
                         self.cache_layer_stride, self.kv_len_out, self.ws, stream)

    def step(self, stream=None):
        self.attn(stream)
        self.lmhead(stream)
        self.compact(stream)

    def status(self):
        return etree_device_status(self.ws)

    def results(self):
        torch.cuda.synchronize()
        return dict(out=self.out.float().cpu(), lse=self.lse.cpu(),
                    accept_len=self.accept_len.cpu().numpy(), path=self.path.cpu().numpy(),
                    out_tokens=self.out_tokens.cpu().numpy(),
                    node_argmax=self.node_argmax.cpu().numpy(),
                    node_gap=self.node_gap.cpu().numpy(), kv_len_out=self.kv_len_out.cpu().numpy())
