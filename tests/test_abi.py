"""C ABI checks that need no GPU: the library loads, exports every entry point the public header
declares, and rejects host-visible argument errors before touching the device."""
import ctypes as C
import os
import re

import pytest

import draft_tree_verification_masked_b200 as et
from draft_tree_verification_masked_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    _build.build()
    return et.lib()


def _declared():
    text = open(os.path.join(ROOT, "include", "etree.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(etree_[a-z_]+)\s*\(", text)))


def test_header_declares_the_three_calls():
    d = _declared()
    for name in ["etree_verify_attn", "etree_lmhead_accept", "etree_kv_compact",
                 "etree_workspace_size", "etree_workspace_init", "etree_device_status",
                 "etree_strerror", "etree_version"]:
        assert name in d


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_version_and_strerror(L):
    assert et.etree_version() == 100
    assert et.etree_strerror(0) == "ok"
    assert "invalid" in et.etree_strerror(-1)
    assert et.etree_strerror(-6).startswith("request cache")


def _batch(B=1, n_total=4, n_max=4, kv_len_max=10, null=False):
    b = et.Batch()
    b.B, b.n_total, b.n_max, b.kv_len_max = B, n_total, n_max, kv_len_max
    fake = None if null else 0x100000
    b.cu_nodes = b.parent = b.tokens = b.kv_len = b.slot_base = b.slot_cap = fake
    return b


FAKE = C.c_void_p(0x100000)


def _attn(L, b, head_dim=128, hq=8, hkv=2, ws_bytes=1 << 20, ws=FAKE):
    return L.etree_verify_attn(C.byref(b), FAKE, FAKE, FAKE, FAKE, FAKE, 100, hq, hkv, head_dim,
                               0.1, FAKE, None, ws, ws_bytes, None)


def test_host_validation_without_a_device(L):
    assert _attn(L, _batch(n_max=65)) == -1
    assert _attn(L, _batch(B=0)) == -1
    assert _attn(L, _batch(n_total=0)) == -1
    assert _attn(L, _batch(null=True)) == -1
    assert _attn(L, _batch(), head_dim=64) == -2
    assert _attn(L, _batch(), hq=6, hkv=4) == -1
    assert _attn(L, _batch(), ws_bytes=16) == -1
    assert _attn(L, _batch(), ws=C.c_void_p(0x100010)) == -1     # not 256-byte aligned
    assert b"aligned" in L.etree_last_error()
    b = _batch()
    assert L.etree_lmhead_accept(C.byref(b), FAKE, FAKE, 100, 1000, 0.0, None, 0, 0, FAKE, FAKE,
                                 FAKE, None, None, FAKE, 1 << 30, None) == -2   # hidden % 64
    assert L.etree_lmhead_accept(C.byref(b), FAKE, FAKE, 128, 1000, 1.0, None, 0, 0, FAKE, FAKE,
                                 FAKE, None, None, FAKE, 1 << 30, None) == -1   # T>0, no q
    assert L.etree_kv_compact(C.byref(b), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 0, 0, 2, 128,
                              C.c_void_p(b.kv_len), FAKE, 1 << 20, None) == -1  # aliasing


def test_workspace_size_grows_with_the_batch(L):
    small = L.etree_workspace_size(C.byref(_batch(B=1, n_total=4)), 8, 2, 128, 1024, 4096)
    big = L.etree_workspace_size(C.byref(_batch(B=64, n_total=1024, n_max=16, kv_len_max=8192)),
                                 40, 8, 128, 5120, 151936)
    assert 256 < small < big
    assert L.etree_workspace_size(C.byref(_batch(B=0)), 8, 2, 128, 1024, 4096) == 0


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "draft_tree_verification_masked_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "liboracle" not in text, f


ALIGNED_WS = C.c_void_p(0x100000)          # 256-byte aligned; never dereferenced: every call
                                           # below fails a host check before any device work
OTHER = C.c_void_p(0x200000)               # a second fake address (outputs that must not alias)


def _rejects(status, code, words):
    """The call failed with `code` and the host message names the failing check."""
    msg = et.lib().etree_last_error()
    assert status == code, (status, msg)
    assert words.encode() in msg, msg


def test_host_validation_of_the_paged_calls(L):
    b = _batch()

    def attn_paged(bt=FAKE, max_pages=4, page=16, num_pages=8, hq=8, hkv=2, head_dim=128):
        return L.etree_verify_attn_paged(C.byref(b), bt, max_pages, page, FAKE, FAKE, FAKE, FAKE,
                                         FAKE, num_pages, hq, hkv, head_dim, 0.1, FAKE, None,
                                         ALIGNED_WS, 1 << 30, None)

    _rejects(attn_paged(bt=None), -1, "block_table")
    _rejects(attn_paged(bt=C.c_void_p(0x100002)), -1, "block_table")    # not 4-byte aligned
    _rejects(attn_paged(max_pages=0), -1, "max_pages")
    for page in (0, 8, 24, 1 << 21):                                     # power of 2, [16, 2^20]
        _rejects(attn_paged(page=page), -1, "page_size")
    _rejects(attn_paged(num_pages=0), -1, "num_pages")
    _rejects(attn_paged(num_pages=1 << 27, page=16), -1, "num_pages")   # 2^31 pool slots
    _rejects(attn_paged(head_dim=64), -2, "head_dim")

    def compact_paged(page=16, num_pages=8, n_layers=1, cache_stride=0, head_dim=128,
                      kv_len_out=OTHER):
        return L.etree_kv_compact_paged(C.byref(b), FAKE, 4, page, FAKE, FAKE, FAKE, FAKE, FAKE,
                                        FAKE, num_pages, n_layers, 4 * 2 * 128, cache_stride, 2,
                                        head_dim, kv_len_out, ALIGNED_WS, 1 << 30, None)

    _rejects(compact_paged(page=12), -1, "page_size")
    _rejects(compact_paged(num_pages=0), -1, "num_pages")
    _rejects(compact_paged(head_dim=96), -2, "head_dim")
    _rejects(compact_paged(n_layers=0), -1, "n_layers")
    _rejects(compact_paged(kv_len_out=FAKE), -1, "aliases")
    # two layers: the cache stride must cover a whole page pool (8 pages x 16 slots x 256)
    _rejects(compact_paged(n_layers=2, cache_stride=8 * 16 * 256 - 8), -1, "page pool")


def test_host_validation_of_the_tree_sampler_and_lm_head(L):
    b = _batch()

    def tree(zbuf=FAKE, rows=4, T=1.0, q=FAKE, hidden_dim=128):
        return L.etree_lmhead_accept_tree(C.byref(b), FAKE, FAKE, hidden_dim, 1000, T, q, 0, 0,
                                          FAKE, FAKE, FAKE, zbuf, rows, ALIGNED_WS, 1 << 30, None)

    _rejects(tree(rows=-1), -1, "zbuf_rows")
    _rejects(tree(zbuf=None, rows=2), -1, "zbuf_rows")
    _rejects(tree(zbuf=C.c_void_p(0x100004)), -1, "zbuf must be 16-byte aligned")
    _rejects(tree(q=None), -1, "q_draft")                                # T > 0 needs draft rows
    for T in (float("nan"), -0.5, float("inf")):
        _rejects(tree(T=T), -1, "temperature")
    _rejects(tree(hidden_dim=96), -2, "hidden_dim")

    def head(hidden=FAKE, vocab=1000, ws=ALIGNED_WS, ws_bytes=1 << 30):
        return L.etree_lmhead_accept(C.byref(b), hidden, FAKE, 128, vocab, 0.0, None, 0, 0, FAKE,
                                     FAKE, FAKE, None, None, ws, ws_bytes, None)

    _rejects(head(vocab=0), -1, "vocab")
    _rejects(head(hidden=None), -1, "NULL")
    _rejects(head(hidden=C.c_void_p(0x100008)), -1, "aligned")          # not 16-byte aligned
    _rejects(head(ws=None), -1, "workspace is NULL")
    _rejects(head(ws_bytes=64), -1, "needs")


def test_host_validation_of_the_attention_scalars(L):
    _rejects(_attn(L, _batch(), hq=130, hkv=2), -1, "hq=130")           # > 64 heads per group
    b = _batch()
    for slots in (0, 1 << 31):
        _rejects(L.etree_verify_attn(C.byref(b), FAKE, FAKE, FAKE, FAKE, FAKE, slots, 8, 2, 128,
                                     0.1, FAKE, None, ALIGNED_WS, 1 << 30, None), -1,
                 "cache_slots")
    _rejects(L.etree_verify_attn(C.byref(b), FAKE, FAKE, FAKE, FAKE, FAKE, 100, 8, 2, 128,
                                 float("nan"), FAKE, None, ALIGNED_WS, 1 << 30, None), -1,
             "scale")
    _rejects(L.etree_verify_attn_noalloc(C.byref(b), FAKE, FAKE, FAKE, FAKE, FAKE, 100, 6, 4, 128,
                                         0.1, FAKE, None, None, None), -1, "hq=6")
    _rejects(_attn(L, _batch(B=2, n_total=1)), -1, "n_total")           # fewer nodes than B


def test_host_validation_of_the_low_rank_head(L):
    def lowrank(hidden=FAKE, M=4, H=128, r=64, V=1000, k=8, ws=ALIGNED_WS, ws_bytes=1 << 30):
        return L.etree_lowrank_candidates(hidden, M, H, FAKE, FAKE, r, FAKE, V, k, FAKE, FAKE,
                                          ws, ws_bytes, None)

    _rejects(lowrank(hidden=None), -1, "NULL")
    _rejects(lowrank(M=0), -1, "M=0")
    for H in (100, 8256):
        _rejects(lowrank(H=H), -2, "hidden_dim")
    for r in (32, 96):
        _rejects(lowrank(r=r), -2, "rank")
    for k, V in ((0, 1000), (17, 1000), (8, 4)):
        _rejects(lowrank(k=k, V=V), -1, "k=")
    _rejects(lowrank(hidden=C.c_void_p(0x100008)), -1, "aligned")
    _rejects(lowrank(ws_bytes=16), -1, "needs")
    assert L.etree_lowrank_workspace_size(0, 128, 64, 1000) == 0
    assert 0 < L.etree_lowrank_workspace_size(4, 128, 64, 1000) < \
        L.etree_lowrank_workspace_size(64, 128, 64, 1000)


def test_host_validation_of_the_status_calls(L):
    _rejects(L.etree_workspace_init(None, 1 << 20, None), -1, "workspace")
    _rejects(L.etree_workspace_init(ALIGNED_WS, 16, None), -1, "workspace")
    _rejects(L.etree_device_status(None, None, None), -1, "workspace")
    for ws, n in ((None, 1 << 20), (C.c_void_p(0x100010), 1 << 20), (ALIGNED_WS, 16)):
        _rejects(L.etree_selftest_timeout(ws, n, None), -1, "workspace")


def test_binding_fails_loudly_without_the_library_or_on_host_memory(tmp_path, monkeypatch):
    """No fallback: a missing library raises on first use, and host tensors are refused before
    any call reaches the library."""
    import torch
    monkeypatch.setattr(et, "_LIB_PATH", str(tmp_path / "libetree.so"))
    monkeypatch.setattr(et, "_lib", None)
    with pytest.raises(et.EtreeError, match="missing"):
        et.lib()
    with pytest.raises(et.EtreeError):
        et.etree_version()
    monkeypatch.undo()
    host = torch.zeros(4, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA device"):
        et.make_batch(host, host, host, host, host.long(), host, 4, 0)
    with pytest.raises(ValueError, match="CUDA device"):
        et.etree_workspace_init(torch.zeros(1024, dtype=torch.uint8))


def test_status_and_detail_codes_agree_across_header_kernels_and_binding():
    """The detail codes the header documents, the kernels' enum and the binding's names list the
    same numbers in the same order; likewise the status codes."""
    hdr = open(os.path.join(ROOT, "include", "etree.h")).read()
    cuh = open(os.path.join(ROOT, "draft_tree_verification_masked_b200", "csrc",
                            "common.cuh")).read()
    det_enum = {int(v): k for k, v in re.findall(r"\b(DET_[A-Z_]+)\s*=\s*(\d+)", cuh)}
    block = hdr[hdr.index("Detail codes:"):hdr.index("etree_device_status(void")]
    det_hdr = {int(n): w.strip() for n, w in re.findall(r"\*\s+(\d+)\s+([a-z_ -]+?)(?::|\n)",
                                                         block)}
    assert sorted(det_enum) == sorted(det_hdr) == sorted(et.DETAIL) == list(range(len(et.DETAIL)))
    assert det_hdr == et.DETAIL
    st_hdr = {int(v): k for k, v in re.findall(r"\b(ETREE_[A-Z]+)\s*=\s*(-?\d+)", hdr)}
    assert st_hdr == {k: v for k, v in et.STATUS.items()}


def test_lm_head_workspace_is_the_documented_regions():
    """Without attention (hq = 0) the workspace is the 256-byte status header plus, each rounded
    up to 256 bytes: LM-head summaries float4 [n_total][2 ceil(V/128)], child token, child logit
    and log2-sum-exp per node, stop row, stop node and offset per request, stop-row hiddens
    bf16 [B][H], draw summaries float4 [B][2 ceil(V/128)], the draw's race floors [B][2],
    arrival counters [B], and per node the child count, logit-row index and parent-row logit."""
    def up(x):
        return (x + 255) // 256 * 256

    for B, nt, H, V in [(1, 16, 1024, 4096), (64, 1024, 5120, 151936), (3, 5, 64, 300)]:
        tiles = 2 * ((V + 127) // 128)
        regions = [nt * tiles * 16, nt * 4, nt * 4, nt * 4, B * 4, B * 4, B * 4, B * H * 2,
                   B * tiles * 16, B * 8, B * 4, nt * 4, nt * 4, nt * 4]
        off = 256
        for r in regions:
            off = up(off + r)
        b = _batch(B=B, n_total=nt, n_max=min(64, nt))
        assert et.lib().etree_workspace_size(C.byref(b), 0, 0, 128, H, V) == off, (B, nt, H, V)
