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
