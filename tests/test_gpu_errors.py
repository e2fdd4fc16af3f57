"""Error behaviour through the C ABI on the GPU: host-visible problems return at once,
device-visible problems set the workspace status word and never trap; the context stays usable.
"""
import pytest
import torch

import draft_tree_verification_masked_b200 as et
from draft_tree_verification_masked_b200 import workload as W
from draft_tree_verification_masked_b200.runner import DeviceStep

pytestmark = pytest.mark.gpu

EINVAL, EUNSUP, EDEVICE, ENOSPACE = -1, -2, -4, -6


def _dev(**kw):
    wl = W.generate("tiny", B=2, kv_len=[100, 300], hidden=256, vocab=512, **kw)
    return wl, DeviceStep(wl)


def _still_works():
    wl, dev = _dev()
    dev.step()
    assert dev.status() == (0, 0)


def test_malformed_parent_sets_device_status():
    """A malformed parent array reports ETREE_EDEVICE (detail 1) and that request is answered
    like any request without a valid tree: nothing accepted, path and tokens all -1 (no bonus
    token that a caller might emit before reading the status); the other request runs."""
    wl, dev = _dev()
    dev.parent[int(wl.cu_nodes[1]) + 3] = 7          # parent not below its child
    dev.accept_len.fill_(7)
    dev.step()
    assert dev.status() == (EDEVICE, 1)
    res = dev.results()
    assert res["accept_len"][1] == 0
    assert (res["path"][1] == -1).all() and (res["out_tokens"][1] == -1).all()
    assert res["out_tokens"][0][int(res["accept_len"][0])] >= 0
    assert dev.status() == (0, 0)                     # read clears
    _still_works()


@pytest.mark.parametrize("T", [0.0, 1.0])
def test_malformed_node_counts_answer_every_request(T):
    """A request with no nodes and one with more than n_max: both report bad node counts and
    accept nothing, with no bonus token, whichever acceptance rule runs."""
    wl = W.generate("tiny", B=3, n_nodes=[5, 9, 6], depth=63, depth_min=63, branch=1,
                    kv_len=[100, 300, 50], hidden=256, vocab=512)
    if T > 0:
        wl.temperature = T
        wl.q_draft = torch.full((wl.n_total, wl.vocab), 1.0 / wl.vocab)
    dev = DeviceStep(wl)
    dev.accept_len.fill_(7)
    dev.cu_nodes[1] = 0                               # request 0: no nodes; request 1: 14 > n_max
    dev.lmhead()
    assert dev.status() == (EDEVICE, 2)
    res = dev.results()
    assert list(res["accept_len"][:2]) == [0, 0]
    assert (res["out_tokens"][:2] == -1).all()
    assert int(res["accept_len"][2]) != 7             # the well-formed request still ran
    _still_works()


@pytest.mark.parametrize("materialize", [False, True])
def test_bad_token_on_a_tree_reports_and_answers_the_request(materialize):
    """A draft token outside [0, vocab) at T > 0 on a branching tree reports ETREE_EDEVICE
    (detail 9) whether the child logits are dot products or read from the materialised rows; that
    request accepts nothing and gets no bonus token (as for a malformed parent), and the other
    one runs."""
    wl = W.generate("tiny", B=2, n_nodes=[7, 9], depth=3, branch=3, kv_len=[100, 300],
                    hidden=256, vocab=512)
    wl.temperature = 1.0
    wl.q_draft = torch.full((wl.n_total, wl.vocab), 1.0 / wl.vocab)
    dev = DeviceStep(wl, tree=True, materialize=materialize)
    dev.accept_len.fill_(7)
    dev.tokens[int(wl.cu_nodes[1]) + 2] = wl.vocab + 3
    dev.lmhead()
    assert dev.status() == (EDEVICE, 9)
    res = dev.results()
    assert res["accept_len"][1] == 0
    assert (res["out_tokens"][1] == -1).all()
    assert res["out_tokens"][0][int(res["accept_len"][0])] >= 0
    _still_works()


def test_bad_page_entry_reports_and_leaves_compaction_untouched():
    wl = W.generate("tiny", B=2, kv_len=[100, 300], hidden=256, vocab=512)
    dev = DeviceStep(wl, page_size=32)
    nump = dev.paged.num_pages
    dev.block_table[1, 2] = nump + 5                  # a used page of request 1, past the pool
    dev.attn()
    assert dev.status() == (EDEVICE, 11)
    dev.block_table[1, 2] = int(dev.paged.block_table[1, 2])
    L1 = int(wl.kv_len[1])
    dev.block_table[1, L1 // 32] = -1                 # request 1's next compaction page
    dev.lmhead()
    dev.compact()
    assert dev.status() == (EDEVICE, 11)
    assert int(dev.kv_len_out[1]) == L1
    _still_works()


def test_kv_len_above_declared_bound():
    wl, dev = _dev()
    dev.kv_len[0] = wl.kv_len_max + 1
    dev.attn()
    assert dev.status() == (EDEVICE, 3)
    _still_works()


def test_cache_capacity_overflow_leaves_request_untouched():
    wl, dev = _dev()
    dev.slot_cap[1] = int(wl.kv_len[1])               # no room for even the root
    before = dev.k_cache.clone()
    dev.step()
    assert dev.status() == (ENOSPACE, 4)
    assert int(dev.kv_len_out[1]) == int(wl.kv_len[1])
    b1 = int(wl.slot_base[1])
    assert torch.equal(dev.k_cache[b1:], before[b1:])
    _still_works()


def test_stochastic_acceptance_on_a_branching_tree_is_unsupported():
    wl = W.generate("tiny", B=2, kv_len=[100, 300], hidden=256, vocab=512)
    wl.temperature = 1.0
    wl.q_draft = torch.full((wl.n_total, wl.vocab), 1.0 / wl.vocab)
    dev = DeviceStep(wl, tree=False)                  # the chain entry point
    dev.lmhead()
    assert dev.status() == (EUNSUP, 5)
    _still_works()


def test_host_argument_errors():
    wl, dev = _dev()
    b = dev.batch
    call = dict(check=False)
    # n_max above 64
    old = b.n_max
    b.n_max = 65
    assert et.etree_verify_attn(b, dev.q, dev.k_tree, dev.v_tree, dev.k_cache, dev.v_cache,
                                dev.scale, dev.out, dev.lse, dev.ws, **call) == EINVAL
    b.n_max = old
    # head_dim 64 is not built
    q64 = torch.zeros(wl.n_total, wl.hq, 64, dtype=torch.bfloat16, device="cuda")
    k64 = torch.zeros(wl.n_total, wl.hkv, 64, dtype=torch.bfloat16, device="cuda")
    assert et.etree_verify_attn(b, q64, k64, k64, dev.k_cache, dev.v_cache, dev.scale,
                                dev.out, dev.lse, dev.ws, **call) == EUNSUP
    # misaligned tensor
    buf = torch.zeros(dev.q.numel() + 8, dtype=torch.bfloat16, device="cuda")
    qm = buf[1:1 + dev.q.numel()].view(dev.q.shape)
    assert qm.data_ptr() % 16 == 2
    assert et.etree_verify_attn(b, qm, dev.k_tree, dev.v_tree, dev.k_cache, dev.v_cache,
                                dev.scale, dev.out, dev.lse, dev.ws, **call) == EINVAL
    # workspace too small
    small = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert et.etree_lmhead_accept(b, dev.hidden, dev.w_lm, 0.0, None, 0, 0, dev.accept_len,
                                  dev.path, dev.out_tokens, None, None, small, **call) == EINVAL
    # negative temperature; T > 0 without draft probabilities
    assert et.etree_lmhead_accept(b, dev.hidden, dev.w_lm, -1.0, None, 0, 0, dev.accept_len,
                                  dev.path, dev.out_tokens, None, None, dev.ws, **call) == EINVAL
    assert et.etree_lmhead_accept(b, dev.hidden, dev.w_lm, 1.0, None, 0, 0, dev.accept_len,
                                  dev.path, dev.out_tokens, None, None, dev.ws, **call) == EINVAL
    # kv_len_out aliasing the batch's kv_len
    assert et.etree_kv_compact(b, dev.accept_len, dev.path, dev.k_tree, dev.v_tree, dev.k_cache,
                               dev.v_cache, 1, 0, 0, dev.kv_len, dev.ws, **call) == EINVAL
    assert dev.status() == (0, 0)
    _still_works()


def test_bounded_wait_runs_out_reports_and_leaves_the_context_usable():
    """A wait that nothing completes, through the library's own bounded wait: it gives up after
    its iteration cap, the status word says ETREE_ETIMEOUT (detail 12), nothing traps, and a normal
    step runs correctly afterwards."""
    import time
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    et.etree_workspace_init(ws)
    t0 = time.perf_counter()
    et.etree_selftest_timeout(ws)
    st, det = et.etree_device_status(ws)
    elapsed = time.perf_counter() - t0
    assert (st, det) == (-5, 12), (st, det)
    assert elapsed < 120.0, elapsed
    assert et.etree_device_status(ws) == (0, 0)           # read clears the word
    _still_works()
