"""The allocation-free attention entry point, checked against the workspace entry point.

etree_verify_attn_noalloc serves callers that cannot allocate device memory (a serving engine
that has reserved HBM for its KV pool, a plugin host without an allocator): its scratch is a
static array inside the library.  This file is collected last so that a failure here does not
stop a fail-fast run before the other tests.  It must pass alone in a fresh process as well as
after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import draft_tree_verification_masked_b200 as et
from draft_tree_verification_masked_b200 import workload as W
from draft_tree_verification_masked_b200.runner import DeviceStep

from . import _parity as P

pytestmark = pytest.mark.gpu


def _noalloc(dev):
    out = torch.full_like(dev.out, float("nan"))
    lse = torch.full_like(dev.lse, float("nan"))
    status = torch.full((2,), -99, dtype=torch.int32, device="cuda")
    et.etree_verify_attn_noalloc(dev.batch, dev.q, dev.k_tree, dev.v_tree, dev.k_cache,
                                 dev.v_cache, dev.scale, out, lse, status)
    torch.cuda.synchronize()
    return out, lse, status.cpu().tolist()


@pytest.mark.parametrize("name", ["tiny", "dense27b_b1"])
def test_noalloc_matches_workspace_entry_point_twice(name):
    wl = W.generate(name)
    dev = DeviceStep(wl)
    plan = et.etree_attn_plan(dev.batch, wl.hq, wl.hkv)
    assert plan["splits"] > 1                       # the static scratch really holds partials
    dev.attn()
    assert dev.status() == (0, 0)
    ref_out, ref_lse = dev.out.clone(), dev.lse.clone()
    for _ in range(2):                              # the second call reuses the array
        out, lse, status = _noalloc(dev)
        assert status == [0, 0]
        diff = (out.float() - ref_out.float()).abs().max().item()
        assert diff <= P.ATTN_MAX_ABS
        assert (lse - ref_lse).abs().max().item() <= P.LSE_ABS
        err = (out.float() - ref_out.float()).cpu().numpy()
        ref = ref_out.float().cpu().numpy()
        assert np.sqrt((err ** 2).mean() / (ref ** 2).mean()) <= P.ATTN_REL_RMS
        assert torch.equal(out, ref_out)            # same kernel, same plan: bit-identical


def test_noalloc_rejects_batches_beyond_the_static_scratch():
    """A 128K-token request with 64 query heads on one KV head splits its keys nine ways: its
    partials need about 19 MB, more than the 16 MiB array.  The call is refused on the host and
    touches nothing; a call with a bad argument is refused the same way."""
    B, n, hq, hkv, L = 1, 64, 64, 1, 131072
    i32 = dict(dtype=torch.int32, device="cuda")
    cu = torch.tensor([0, n], **i32)
    parent = torch.tensor([-1] + list(range(n - 1)), **i32)
    tokens = torch.zeros(n, **i32)
    kv_len = torch.full((B,), L, **i32)
    slot_cap = torch.full((B,), L + 64, **i32)
    slot_base = torch.zeros(B, dtype=torch.int64, device="cuda")
    batch = et.make_batch(cu, parent, tokens, kv_len, slot_base, slot_cap, n, L)
    bf = dict(dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(n, hq, 128, **bf)
    kt = torch.zeros(n, hkv, 128, **bf)
    kc = torch.zeros(L + 64, hkv, 128, **bf)
    out = torch.full((n, hq, 128), 7.0, **bf)
    need = et.etree_workspace_size(batch, hq, hkv, 128, 0, 0)
    assert need > 16 << 20
    st = et.etree_verify_attn_noalloc(batch, q, kt, kt, kc, kc, 0.088, out, None, check=False)
    assert st == -1
    assert b"static array" in et.lib().etree_last_error()
    st = et.etree_verify_attn_noalloc(batch, q, kt, kt, kc, kc, float("nan"), out, None,
                                      check=False)
    assert st == -1
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
