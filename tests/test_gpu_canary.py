"""Out-of-bounds writes: every buffer the library writes -- outputs, the logit rows of branching
nodes, the workspace -- is handed over as a view into a larger buffer whose head and tail hold a
sentinel pattern.  After a full step the padding must be intact, and the results must still match
the oracle (so the views were used, not stale copies)."""
import pytest
import torch

from draft_tree_verification_masked_b200 import workload as W
from draft_tree_verification_masked_b200.runner import DeviceStep

from . import _parity as P

pytestmark = pytest.mark.gpu

PAD = 4096                      # bytes of sentinel before and after each buffer
SENTINEL = 0xA5


def _guard(t: torch.Tensor):
    """A view with t's shape and dtype inside a sentinel-padded byte buffer."""
    nbytes = t.numel() * t.element_size()
    big = torch.full((nbytes + 2 * PAD,), SENTINEL, dtype=torch.uint8, device=t.device)
    view = big[PAD:PAD + nbytes].view(t.dtype).view(t.shape)
    view.copy_(t)
    return big, view


def _intact(big: torch.Tensor) -> bool:
    head, tail = big[:PAD], big[-PAD:]
    return bool((head == SENTINEL).all()) and bool((tail == SENTINEL).all())


def _guarded_step(wl, **kw):
    dev = DeviceStep(wl, **kw)
    bigs = {}
    for name in ("out", "lse", "node_argmax", "node_gap", "kv_len_out", "accept_len", "path",
                 "out_tokens", "ws") + (("zbuf",) if dev.zbuf is not None else ()):
        bigs[name], view = _guard(getattr(dev, name))
        setattr(dev, name, view)
    dev.step()
    st, det = dev.status()
    assert st == 0, (st, det)
    torch.cuda.synchronize()
    for name, big in bigs.items():
        assert _intact(big), f"write outside {name}"
    return dev, dev.results()


def test_greedy_step_stays_inside_its_buffers():
    wl = W.generate("tiny", B=5, n_nodes=[1, 4, 16, 33, 64], kv_len=[0, 7, 63, 64, 300],
                    depth=8, depth_min=1, branch=None, width=16, hidden=512, vocab=4096 + 5)
    dev, res = _guarded_step(wl)
    P.attn_compare(wl, dev)
    excused, near, ores = P.greedy_compare(wl, res, list(range(wl.B)))
    P.compact_compare(wl, dev, ores, list(range(wl.B)), excused)
    assert near <= 1


def test_stochastic_chain_step_stays_inside_its_buffers():
    wl = W.generate("conc512", B=11, n_nodes=[4, 5, 6, 1, 2, 4, 4, 3, 2, 1, 4], depth=5,
                    depth_min=5, kv_len=(20, 400), hidden=512, vocab=4096 + 3, temperature=1.0)
    dev, res = _guarded_step(wl, tree=False)
    excused, near, ores = P.chain_compare(wl, res, list(range(wl.B)))
    P.compact_compare(wl, dev, ores, list(range(wl.B)), excused)
    assert near <= 2


def test_branching_tree_step_stays_inside_its_buffers():
    wl = W.generate("tree64_t1", B=6, n_nodes=[16, 5, 1, 12, 9, 3], depth=4, depth_min=2,
                    branch=4, kv_len=(20, 400), hidden=512, vocab=4096 + 3, temperature=1.0)
    dev, res = _guarded_step(wl)
    assert dev.tree and dev.zbuf is not None
    excused, near, ores = P.tree_compare(wl, res, list(range(wl.B)))
    P.compact_compare(wl, dev, ores, list(range(wl.B)), excused)
    assert near <= 2


def test_paged_step_stays_inside_its_buffers():
    wl = W.generate("tiny", B=4, n_nodes=[3, 16, 1, 9], kv_len=[5, 200, 0, 77], hidden=512,
                    vocab=2048)
    dev, res = _guarded_step(wl, page_size=16)
    P.attn_compare_paged(wl, dev)
    excused, near, ores = P.greedy_compare(wl, res, list(range(wl.B)))
    P.compact_compare_paged(wl, dev, ores, list(range(wl.B)), excused)
    assert near <= 1
