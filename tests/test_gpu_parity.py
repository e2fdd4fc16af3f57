"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the same seeded inputs.

Every workload is compared at full size, in the launch configuration the benchmark times: every
request's acceptance outputs, compacted rows and every attention row.  Other launch plans (KV
split counts, 32- and 64-key tiles, LM-head row tiles) are reached through the shapes that make
the library's planner choose them, which etree_attn_plan reports.

Near-ties (a decision that the fp32 and fp64 arithmetic can legitimately take differently:
a top-1 / top-2 logit gap under 1e-3 at T = 0, a sampling comparison within rounding at T > 0)
are replayed, counted and logged in the session summary.  Each test allows at most one excused
request: the chance of even one is about 1e-5 per decision (an argmax flips only when the gap is
within the fp32 error of the logits, a few 1e-6; a sampling decision only when the fp64
quantities it compares agree to 1e-5), far below one per test.
"""
import dataclasses

import numpy as np
import pytest
import torch

import draft_tree_verification_masked_b200 as et
from draft_tree_verification_masked_b200 import workload as W
from draft_tree_verification_masked_b200.runner import DeviceStep

from . import _parity as P

pytestmark = pytest.mark.gpu

MAX_EXCUSED = 1


def _run(wl, n_layers=1, **kw):
    dev = DeviceStep(wl, n_layers=n_layers, **kw)
    dev.step()
    st, det = dev.status()
    assert st == 0, (st, det)
    return dev, dev.results()


def _accept_check(wl, dev, res, reqs, label):
    if wl.temperature == 0.0:
        excused, near, ores = P.greedy_compare(wl, res, reqs)
    elif dev.tree:
        excused, near, ores = P.tree_compare(wl, res, reqs)
    else:
        excused, near, ores = P.chain_compare(wl, res, reqs)
    P.log_near(label, wl, res, ores, reqs, near)
    assert near <= MAX_EXCUSED, near
    return excused, ores


def _full_check(wl, attn_rows=None, requests=None, label=None, **kw):
    dev, res = _run(wl, **kw)
    P.attn_compare(wl, dev, rows=attn_rows)
    reqs = list(range(wl.B)) if requests is None else requests
    excused, ores = _accept_check(wl, dev, res, reqs, label or wl.name)
    P.compact_compare(wl, dev, ores, reqs, excused)
    return dev, res


def _plan(wl, kv_len_max=None):
    dev_batch = DeviceStep(wl, kv_len_max=kv_len_max).batch
    return et.etree_attn_plan(dev_batch, wl.hq, wl.hkv)


def test_tiny_config():
    _full_check(W.generate("tiny"))


def test_dense27b_single_request_full_size():
    _full_check(W.generate("dense27b_b1"))


@pytest.mark.parametrize("name", ["long32k", "long128k"])
def test_long_context(name):
    _full_check(W.generate(name))


def test_batch64():
    _full_check(W.generate("batch64"))


def test_conc512_stochastic_chains():
    _full_check(W.generate("conc512"))


def test_ragged_trees_and_lengths():
    wl = W.generate("tiny", B=6, n_nodes=[1, 4, 16, 33, 64, 2], kv_len=[0, 1, 63, 64, 65, 200],
                    depth=8, depth_min=1, branch=None, width=16, vocab=4096 + 128 + 5,
                    hidden=1024)
    _full_check(wl)


@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 2), (32, 1), (12, 4)])
def test_gqa_group_sizes(hq, hkv):
    wl = W.generate("tiny", B=3, hq=hq, hkv=hkv, kv_len=(100, 700), hidden=512, vocab=2048)
    _full_check(wl)


def test_chain_of_64_and_single_node():
    wl = W.generate("tiny", B=2, n_nodes=[64, 1], depth=63, depth_min=63, branch=1,
                    kv_len=[300, 5], hidden=256, vocab=1000)
    _full_check(wl)


# KV lengths of a two-request tiny batch (16-node trees, 2 KV heads) whose plan splits the keys
# 1, 2, 3 and 7 ways (64-key tiles: tiles = ceil(L / 64) + 1, splits = min(37, tiles / 4)).
@pytest.mark.parametrize("nsplit,kv", [(1, [300, 100]), (2, [500, 64]), (3, [800, 333]),
                                       (7, [1700, 1000])])
def test_split_count_does_not_change_results(nsplit, kv):
    wl = W.generate("tiny", B=2, kv_len=kv, hidden=256, vocab=512)
    assert _plan(wl)["splits"] == nsplit
    _full_check(wl)


def test_many_row_tiles_and_ragged_vocab():
    wl = W.generate("tiny", B=9, kv_len=(10, 300), hidden=1024, vocab=4096 + 200)
    assert wl.n_total > 128
    _full_check(wl)


@pytest.mark.parametrize("T", [1.0, 0.6])
def test_stochastic_chains_small(T):
    wl = W.generate("conc512", B=37, n_nodes=[4, 5, 6, 1, 2] * 7 + [4, 4], depth=5,
                    depth_min=5, kv_len=(20, 400), hidden=512, vocab=4096 + 3, temperature=T)
    _full_check(wl)


def test_repeat_is_bitwise_deterministic():
    wl = W.generate("tiny", B=3, kv_len=(100, 900), hidden=512, vocab=2048)
    dev = DeviceStep(wl)
    dev.step()
    first = dev.results()
    dev.step()
    second = dev.results()
    for k in first:
        a, b = first[k], second[k]
        if isinstance(a, torch.Tensor):
            assert torch.equal(a, b), k
        else:
            assert np.array_equal(a, b), k


def test_multi_layer_compaction_against_oracle():
    """Host-built accept lengths and paths, 5 layers with distinct contents, ragged requests."""
    import oracle
    wl = W.generate("tiny", B=5, n_nodes=[1, 4, 16, 33, 64], kv_len=[0, 7, 63, 64, 65],
                    depth=8, depth_min=1, branch=None, width=16, hidden=256, vocab=512)
    L = 5
    g = np.random.default_rng(3)
    a = np.array([0, 3, 5, 1, 63], dtype=np.int32)
    path = np.full((wl.B, 64), -1, dtype=np.int32)
    for r in range(wl.B):
        n = wl.nodes(r)
        path[r, 0] = 0
        path[r, 1:a[r] + 1] = g.choice(np.arange(1, n), a[r], replace=False)
    dev = DeviceStep(wl, n_layers=L)
    kt = (torch.randn(L, wl.n_total, wl.hkv, 128) * 3).to(torch.bfloat16)
    vt = (torch.randn(L, wl.n_total, wl.hkv, 128) * 3).to(torch.bfloat16)
    kc = torch.randn(L, wl.slots, wl.hkv, 128).to(torch.bfloat16)
    vc = torch.randn(L, wl.slots, wl.hkv, 128).to(torch.bfloat16)
    dev.kt_layers.copy_(kt)
    dev.vt_layers.copy_(vt)
    dev.kc_layers.copy_(kc)
    dev.vc_layers.copy_(vc)
    dev.accept_len.copy_(torch.from_numpy(a))
    dev.path.copy_(torch.from_numpy(path))
    dev.compact()
    assert dev.status()[0] == 0
    ek, ev = oracle._u16(kc).copy(), oracle._u16(vc).copy()
    st, newlen = oracle.kv_compact(wl.cu_nodes, wl.kv_len, wl.slot_base, wl.slot_cap, a, path,
                                   kt, vt, ek, ev, L, wl.n_total * wl.hkv * 128,
                                   wl.slots * wl.hkv * 128, wl.hkv, 128)
    assert st == 0
    assert np.array_equal(oracle._u16(dev.kc_layers.cpu()), ek)
    assert np.array_equal(oracle._u16(dev.vc_layers.cpu()), ev)
    assert np.array_equal(dev.kv_len_out.cpu().numpy(), newlen)


@pytest.mark.parametrize("case", ["ragged", "g1", "g8_chain", "conc_like", "two_blocks"])
def test_attention_32key_tiles(case):
    """The 32-key, two-CTAs-per-SM attention shape (chosen for 64K or more cached keys: here a
    loose kv_len_max bound asks for it): two tree tiles for trees over 32 nodes, lane-quarter
    rotation of small row blocks, ragged lengths, splits with nothing to do."""
    if case == "ragged":
        wl = W.generate("tiny", B=6, n_nodes=[1, 4, 16, 33, 64, 2],
                        kv_len=[0, 1, 31, 32, 33, 200], depth=8, depth_min=1, branch=None,
                        width=16, vocab=1000, hidden=256)
    elif case == "g1":
        wl = W.generate("tiny", B=3, hq=8, hkv=8, kv_len=(100, 700), hidden=256, vocab=512)
    elif case == "g8_chain":
        wl = W.generate("tiny", B=2, hq=16, hkv=2, n_nodes=[40, 7], depth=39, depth_min=39,
                        branch=1, kv_len=[95, 1], hidden=256, vocab=512)
    elif case == "conc_like":
        wl = W.generate("conc512", B=9, hq=10, hkv=2, kv_len=(30, 300), hidden=256, vocab=512)
    else:
        wl = W.generate("tiny", B=2, hq=40, hkv=8, n_nodes=[64, 30], depth=8, depth_min=8,
                        branch=None, width=16, kv_len=[500, 77], hidden=256, vocab=512)
    assert _plan(wl, kv_len_max=65536)["rows_per_cta"] > 0
    _full_check(wl, kv_len_max=65536)


def test_attention_32key_tiles_from_many_work_items():
    """The other route to 32-key tiles: at least one (request, KV head, row block) per SM."""
    wl = W.generate("tiny", B=80, n_nodes=[1, 3, 5, 8] * 20, depth=4, depth_min=2, branch=None,
                    width=16, kv_len=(0, 200), hidden=256, vocab=512)
    assert _plan(wl)["splits"] >= 1 and wl.B * wl.hkv >= 148
    _full_check(wl)


@pytest.mark.parametrize("rows", [64, 100, 200])
@pytest.mark.parametrize("T", [0.0, 1.0])
def test_lmhead_row_tile_heights(rows, T):
    """Up to 64 rows the LM head runs M=64 MMAs (rows 16q..16q+15 in the first half of TMEM
    lane quarter q); up to 128 rows one M=128 row tile; with more row tiles the summaries are
    per vocab tile instead of per CTA.  All must give the oracle's results."""
    sizes = {64: [20, 1, 31, 12], 100: [20, 1, 31, 12, 36], 200: [20, 1, 31, 12, 36, 50, 50]}[rows]
    shape = dict(depth=6, depth_min=4, branch=None, width=16) if T == 0.0 else \
        dict(depth=63, depth_min=63, branch=1)            # sampling verifies chains
    wl = W.generate("tiny", B=len(sizes), n_nodes=sizes, kv_len=(50, 400), hidden=512,
                    vocab=8192 + 77, temperature=T, **shape)
    assert wl.n_total == rows
    _full_check(wl)


# ------------------------------------------------------------ T > 0 on branching trees
def _branching(T, vocab, B=9, seed_nodes=(16, 5, 1, 12, 9, 3, 16, 7, 2)):
    return W.generate("tree64_t1", B=B, n_nodes=list(seed_nodes[:B]), depth=4, depth_min=2,
                      branch=4, kv_len=(20, 400), hidden=512, vocab=vocab, temperature=T)


@pytest.mark.parametrize("T,vocab", [(1.0, 4096 + 3), (0.6, 8192), (1.6, 2048 + 128)])
def test_stochastic_branching_trees(T, vocab):
    """Multi-candidate acceptance: sibling rejections with residual passes over materialised
    logit rows, ragged and aligned vocab sizes (scalar and float4 paths)."""
    wl = _branching(T, vocab)
    dev, res = _full_check(wl)
    assert dev.tree and dev.zbuf is not None


def test_tree_sampler_on_chains_matches_chain_rule():
    """The branching-tree entry point on chains (no logit rows needed) gives the chain rule."""
    wl = W.generate("conc512", B=37, n_nodes=[4, 5, 6, 1, 2] * 7 + [4, 4], depth=5,
                    depth_min=5, kv_len=(20, 400), hidden=512, vocab=4096 + 3, temperature=1.0)
    dev, res = _run(wl, tree=True)
    assert dev.zbuf is None
    excused, near, ores = P.chain_compare(wl, res, list(range(wl.B)))
    P.log_near("tree_entry_on_chains", wl, res, ores, list(range(wl.B)), near)
    assert near <= MAX_EXCUSED


def test_tree64_t1_full_size():
    _full_check(W.generate("tree64_t1"))


@pytest.mark.parametrize("name", ["conc512", "tree64_t1"])
def test_materialised_draw_full_size(name):
    """Every row's logits kept (zbuf of n_total rows): the bonus draw reads the stop rows there
    instead of a second pass over W, chains and branching trees alike."""
    wl = W.generate(name)
    dev, res = _full_check(wl, materialize=True, label=f"{name}_materialised")
    assert dev.tree and dev.zbuf.shape[0] == wl.n_total
    _stored_logits_check(wl, dev)


def _stored_logits_check(wl, dev, nrows=40):
    """The stored rows are the logits themselves (fp32 accumulation of bf16 products over the
    hidden size: within 1e-3 (1 + |z|) of fp64), each in its own row, on sampled rows including
    the first and last (row tiles and vocab tails)."""
    import oracle
    g = np.random.default_rng(7)
    rows = np.unique(np.concatenate([[0, wl.n_total - 1],
                                     g.integers(0, wl.n_total, nrows)])).astype(np.int32)
    z = oracle.logits(wl.hidden, wl.w_lm, rows)
    got = dev.zbuf[torch.as_tensor(rows, dtype=torch.long, device=dev.zbuf.device)].cpu().numpy()
    assert np.all(np.abs(got - z) <= 1e-3 * (1.0 + np.abs(z))), float(np.abs(got - z).max())


@pytest.mark.parametrize("T", [1.0, 0.6])
def test_materialised_draw_small(T):
    wl = W.generate("conc512", B=37, n_nodes=[4, 5, 6, 1, 2] * 7 + [4, 4], depth=5,
                    depth_min=5, kv_len=(20, 400), hidden=512, vocab=4096 + 3, temperature=T)
    dev, _ = _full_check(wl, materialize=True)
    _stored_logits_check(wl, dev)
    wl = _branching(T, 8192 + 4)
    dev, _ = _full_check(wl, materialize=True)
    _stored_logits_check(wl, dev)
    wl = _branching(T, 8192 + 5)                          # vocab not a multiple of 4: direct stores
    dev, _ = _full_check(wl, materialize=True)
    _stored_logits_check(wl, dev)


def test_logit_buffer_overflow_reports_and_answers_the_rest():
    """Fewer logit rows than branching nodes: ETREE_ENOSPACE (detail 10); the requests whose
    branching nodes all got a row still match the oracle, the others accept nothing."""
    from draft_tree_verification_masked_b200.runner import branching_nodes
    wl = _branching(1.0, 4096 + 3)
    need = branching_nodes(wl)
    dev = DeviceStep(wl, zbuf_rows=need // 2)
    dev.lmhead()
    assert dev.status() == (-6, 10)
    res = dev.results()
    # rows are assigned in node order: request r keeps its rows iff all of its branching nodes
    # come before the cut
    cnt, got = 0, []
    for r in range(wl.B):
        a0, a1 = int(wl.cu_nodes[r]), int(wl.cu_nodes[r + 1])
        kids = np.bincount(wl.parent[a0 + 1:a1], minlength=a1 - a0)
        cnt += int((kids >= 2).sum())
        if cnt <= need // 2:
            got.append(r)
        else:
            assert res["accept_len"][r] == 0 and res["out_tokens"][r][0] >= 0   # root draw only
    excused, near, ores = P.tree_compare(wl, res, got)
    assert near <= MAX_EXCUSED


# ------------------------------------------------------------------------- paged KV caches
def _paged_check(wl, page_size, attn_rows=None, requests=None, **kw):
    dev, res = _run(wl, page_size=page_size, **kw)
    P.attn_compare_paged(wl, dev, rows=attn_rows)
    reqs = list(range(wl.B)) if requests is None else requests
    excused, ores = _accept_check(wl, dev, res, reqs, f"{wl.name}@p{page_size}")
    P.compact_compare_paged(wl, dev, ores, reqs, excused)
    return dev, res


@pytest.mark.parametrize("page_size", [16, 32, 64, 256])
@pytest.mark.parametrize("keys", [32, 64])
def test_paged_cache(page_size, keys):
    """Pages smaller than, equal to and larger than the key tile, both tile shapes (32-key tiles
    through a loose kv_len_max bound), ragged lengths including an empty cache and lengths that
    end mid-page."""
    wl = W.generate("tiny", B=6, n_nodes=[1, 4, 16, 33, 64, 2],
                    kv_len=[0, 1, 31, 64, 65, 700], depth=8, depth_min=1, branch=None,
                    width=16, vocab=1000, hidden=256)
    _paged_check(wl, page_size, kv_len_max=65536 if keys == 32 else None)


def test_paged_cache_splits_and_stochastic_chains():
    wl = W.generate("conc512", B=9, kv_len=(30, 900), hidden=256, vocab=512)
    assert _plan(wl)["splits"] > 1
    _paged_check(wl, 16)


def test_batch64_paged16_full_size():
    _paged_check(W.generate("batch64"), 16)


# -------------------------------------------------------------------- low-rank candidate head
def _lowrank_run(lw):
    from draft_tree_verification_masked_b200 import (etree_lowrank_candidates,
                                                     etree_lowrank_workspace_size,
                                                     etree_workspace_init, etree_device_status)
    dev = torch.device("cuda")
    h, D, U, Wt = (x.to(dev) for x in (lw.hidden, lw.D, lw.U, lw.W))
    ws = torch.zeros(etree_lowrank_workspace_size(lw.M, lw.H, lw.r, lw.V), dtype=torch.uint8,
                     device=dev)
    etree_workspace_init(ws)
    ids = torch.full((lw.M, lw.k), -7, dtype=torch.int32, device=dev)
    lg = torch.empty(lw.M, lw.k, dtype=torch.float32, device=dev)
    etree_lowrank_candidates(h, D, U, Wt, lw.k, ids, lg, ws)
    assert etree_device_status(ws) == (0, 0)
    return ids.cpu().numpy(), lg.cpu().numpy()


@pytest.mark.parametrize("over", [dict(), dict(k=16), dict(k=1), dict(r=128, k=5),
                                  dict(M=130, V=3000, k=12), dict(M=64, V=20000, r=192, k=16)])
def test_lowrank_candidates_small(over):
    lw = W.lowrank("lowrank_tiny", **over)
    ids, lg = _lowrank_run(lw)
    P.lowrank_compare(lw, ids, lg)


def test_lowrank_select_beyond_the_register_entries():
    """Two row tiles make the screen keep lists per vocab tile: at V = 60,000 a row has more than
    8,192 list entries, so the select reads the rest of them again in every pass."""
    lw = W.lowrank("lowrank_tiny", M=130, V=60000, k=16)
    ids, lg = _lowrank_run(lw)
    P.lowrank_compare(lw, ids, lg)


def test_lowrank_select_takes_the_lowest_ids_of_a_shared_value():
    """Forty vocab ids spread over the vocabulary (so over different CTAs' lists) share one U
    row, scaled by 8 so that it dominates the rows where it scores positive: there more than k
    ids tie for the largest screen values, bit for bit, and the select must take the lowest of
    them.  Checked directly on the GPU's sets and against the oracle."""
    lw = W.lowrank("lowrank_tiny", M=32, V=20000, k=16)
    U = lw.U.clone()
    group = [37 + 487 * i for i in range(40)]
    U[group] = (U[5].float() * 8).to(torch.bfloat16)
    lw = dataclasses.replace(lw, U=U)
    ids, lg = _lowrank_run(lw)
    gset = set(group)
    full = 0
    for m in range(lw.M):
        sel = sorted(c for c in ids[m].tolist() if c in gset)
        assert sel == group[:len(sel)], (m, sel)
        full += len(sel) == lw.k
    assert full >= 1                                   # some rows cut through the tie
    P.lowrank_compare(lw, ids, lg)


@pytest.mark.parametrize("name", ["lowrank_r512", "lowrank_r128"])
def test_lowrank_candidates_full_size(name):
    lw = W.lowrank(name)
    ids, lg = _lowrank_run(lw)
    P.lowrank_compare(lw, ids, lg)


def test_inputs_written_by_the_kernel_before_each_call():
    """Every input a call reads is produced by the kernel launched just before it on the same
    stream (device-to-device copies from a scrambled start), as a model's layers would produce
    them.  The calls start their set-up early (programmatic dependent launch) and must still see
    the finished inputs: the results match the oracle."""
    wl = W.generate("tiny")
    dev = DeviceStep(wl)
    good = dev.inputs.buf.clone()
    hid, q = dev.hidden.clone(), dev.q.clone()
    for _ in range(3):
        dev.inputs.buf.copy_(good)
        dev.q.zero_()
        dev.hidden.zero_()
        torch.cuda.synchronize()
        dev.q.copy_(q)                                   # written right before the attention
        dev.attn()
        dev.hidden.copy_(hid)                            # written right before the LM head
        dev.lmhead()
        dev.compact()
        st, det = dev.status()
        assert st == 0, (st, det)
    res = dev.results()
    P.attn_compare(wl, dev)
    excused, near, ores = P.greedy_compare(wl, res, list(range(wl.B)))
    P.compact_compare(wl, dev, ores, list(range(wl.B)), excused)
    assert near <= 1, near


def test_lowrank_hidden_written_by_the_kernel_before_the_call():
    """The hidden rows are produced by the kernel launched just before the low-rank call on the
    same stream (its kernels start their set-up early under programmatic dependent launch), and
    the call repeats on the same workspace: the candidates still match the oracle."""
    from draft_tree_verification_masked_b200 import (etree_lowrank_candidates,
                                                     etree_lowrank_workspace_size,
                                                     etree_workspace_init, etree_device_status)
    lw = W.lowrank("lowrank_tiny")
    dev = torch.device("cuda")
    h, D, U, Wt = (x.to(dev) for x in (lw.hidden, lw.D, lw.U, lw.W))
    ws = torch.zeros(etree_lowrank_workspace_size(lw.M, lw.H, lw.r, lw.V), dtype=torch.uint8,
                     device=dev)
    etree_workspace_init(ws)
    ids = torch.full((lw.M, lw.k), -7, dtype=torch.int32, device=dev)
    lg = torch.empty(lw.M, lw.k, dtype=torch.float32, device=dev)
    h_in = torch.zeros_like(h)
    for _ in range(3):
        h_in.zero_()
        torch.cuda.synchronize()
        h_in.copy_(h)                                    # written right before the call
        etree_lowrank_candidates(h_in, D, U, Wt, lw.k, ids, lg, ws)
    assert etree_device_status(ws) == (0, 0)
    P.lowrank_compare(lw, ids.cpu().numpy(), lg.cpu().numpy())
