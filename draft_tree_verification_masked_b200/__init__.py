"""etree -- target-model verification of a draft token tree on NVIDIA B200 (sm_100a).

Thin ctypes binding of ``libetree.so``; argument marshalling only.  Every step of the
computation runs in the library's CUDA kernels.  PyTorch supplies device memory and streams.
The binding never falls back to anything else: without the built library (or without a CUDA
device) every entry point raises.

Entry points (same names as the C ABI in ``include/etree.h``)::

    etree_workspace_size(batch, hq, hkv, head_dim, hidden_dim, vocab) -> int
    etree_workspace_init(workspace, stream=None)
    etree_verify_attn(batch, q, k_tree, v_tree, k_cache, v_cache, scale, out, lse, workspace)
    etree_lmhead_accept(batch, hidden, w_lm, temperature, q_draft, seed, step, accept_len, path,
                        out_tokens, node_argmax, node_gap, workspace)
    etree_lmhead_accept_tree(batch, hidden, w_lm, temperature, q_draft, seed, step, accept_len,
                             path, out_tokens, zbuf, workspace)
    etree_kv_compact(batch, accept_len, path, k_tree, v_tree, k_cache, v_cache, n_layers,
                     tree_layer_stride, cache_layer_stride, kv_len_out, workspace)
    etree_device_status(workspace, stream=None) -> (status, detail)
"""
from __future__ import annotations

import ctypes as C
import os

import torch

__all__ = [
    "EtreeError", "Batch", "make_batch", "lib", "library_path", "etree_workspace_size",
    "etree_workspace_init", "etree_verify_attn", "etree_verify_attn_noalloc",
    "etree_lmhead_accept", "etree_lmhead_accept_tree", "etree_lmhead_accept_timed",
    "etree_kv_compact",
    "etree_verify_attn_paged", "etree_kv_compact_paged", "etree_verify_cost", "etree_plan_tree",
    "cost_table", "load_cost_table", "etree_lowrank_workspace_size",
    "etree_lowrank_candidates", "etree_device_status", "etree_selftest_timeout", "etree_strerror",
    "etree_version", "etree_attn_plan", "STATUS",
]

HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(HERE, "libetree.so")

STATUS = {0: "ETREE_OK", -1: "ETREE_EINVAL", -2: "ETREE_EUNSUPPORTED", -3: "ETREE_ECUDA",
          -4: "ETREE_EDEVICE", -5: "ETREE_ETIMEOUT", -6: "ETREE_ENOSPACE"}
DETAIL = {0: "none", 1: "bad parent", 2: "bad node count", 3: "bad kv_len", 4: "capacity",
          5: "not a chain", 6: "bad path", 7: "attention wait", 8: "gemm wait", 9: "bad token",
          10: "logit rows", 11: "bad page", 12: "self-test wait", 13: "walk wait"}

EXPORTS = ["etree_workspace_size", "etree_workspace_init", "etree_verify_attn",
           "etree_verify_attn_paged", "etree_kv_compact_paged", "etree_verify_cost",
           "etree_plan_tree", "etree_lowrank_workspace_size", "etree_lowrank_candidates",
           "etree_lmhead_accept", "etree_lmhead_accept_tree", "etree_lmhead_accept_timed",
           "etree_kv_compact", "etree_device_status", "etree_strerror",
           "etree_version", "etree_last_error", "etree_attn_plan", "etree_verify_attn_noalloc",
           "etree_selftest_timeout"]


class EtreeError(RuntimeError):
    def __init__(self, status: int, msg: str = ""):
        self.status = status
        super().__init__(f"{STATUS.get(status, status)}: {msg}")


class Batch(C.Structure):
    _fields_ = [("B", C.c_int32), ("n_total", C.c_int32), ("n_max", C.c_int32),
                ("kv_len_max", C.c_int32), ("cu_nodes", C.c_void_p), ("parent", C.c_void_p),
                ("tokens", C.c_void_p), ("kv_len", C.c_void_p), ("slot_base", C.c_void_p),
                ("slot_cap", C.c_void_p)]


_lib = None


def library_path() -> str:
    return _LIB_PATH


def lib():
    """Load libetree.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise EtreeError(-3, f"{_LIB_PATH} is missing: run `python -m "
                             "draft_tree_verification_masked_b200._build` first")
    L = C.CDLL(_LIB_PATH)
    vp, i32, i64, u64, f32 = C.c_void_p, C.c_int32, C.c_int64, C.c_uint64, C.c_float
    bp = C.POINTER(Batch)
    L.etree_workspace_size.argtypes = [bp, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int]
    L.etree_workspace_size.restype = C.c_size_t
    L.etree_workspace_init.argtypes = [vp, C.c_size_t, vp]
    L.etree_workspace_init.restype = C.c_int
    L.etree_verify_attn.argtypes = [bp, vp, vp, vp, vp, vp, i64, C.c_int, C.c_int, C.c_int, f32,
                                    vp, vp, vp, C.c_size_t, vp]
    L.etree_verify_attn.restype = C.c_int
    L.etree_lmhead_accept.argtypes = [bp, vp, vp, C.c_int, C.c_int, f32, vp, u64, u64, vp, vp,
                                      vp, vp, vp, vp, C.c_size_t, vp]
    L.etree_lmhead_accept.restype = C.c_int
    L.etree_lmhead_accept_tree.argtypes = [bp, vp, vp, C.c_int, C.c_int, f32, vp, u64, u64, vp,
                                           vp, vp, vp, C.c_int32, vp, C.c_size_t, vp]
    L.etree_lmhead_accept_tree.restype = C.c_int
    L.etree_lmhead_accept_timed.argtypes = [bp, vp, vp, C.c_int, C.c_int, f32, vp, u64, u64, vp,
                                            vp, vp, vp, vp, vp, C.c_int32, C.c_int32,
                                            C.POINTER(C.c_void_p), vp, C.c_size_t, vp]
    L.etree_lmhead_accept_timed.restype = C.c_int
    L.etree_kv_compact.argtypes = [bp, vp, vp, vp, vp, vp, vp, C.c_int, i64, i64, C.c_int,
                                   C.c_int, vp, vp, C.c_size_t, vp]
    L.etree_kv_compact.restype = C.c_int
    L.etree_verify_attn_paged.argtypes = [bp, vp, C.c_int32, C.c_int32, vp, vp, vp, vp, vp, i64,
                                          C.c_int, C.c_int, C.c_int, f32, vp, vp, vp, C.c_size_t,
                                          vp]
    L.etree_verify_attn_paged.restype = C.c_int
    L.etree_lowrank_workspace_size.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int]
    L.etree_lowrank_workspace_size.restype = C.c_size_t
    L.etree_lowrank_candidates.argtypes = [vp, C.c_int, C.c_int, vp, vp, C.c_int, vp, C.c_int,
                                           C.c_int, vp, vp, vp, C.c_size_t, vp]
    L.etree_lowrank_candidates.restype = C.c_int
    L.etree_verify_cost.argtypes = [C.POINTER(CostTable), C.c_double, C.c_double, C.c_double,
                                    C.POINTER(C.c_double)]
    L.etree_verify_cost.restype = C.c_int
    L.etree_plan_tree.argtypes = [C.POINTER(CostTable), C.c_int32, C.c_int32,
                                  C.POINTER(C.c_float), C.c_int32, C.c_float, C.c_float,
                                  C.c_int32, C.c_int32, C.c_int32, C.POINTER(TreePlan)]
    L.etree_plan_tree.restype = C.c_int
    L.etree_kv_compact_paged.argtypes = [bp, vp, C.c_int32, C.c_int32, vp, vp, vp, vp, vp, vp,
                                         i64, C.c_int, i64, i64, C.c_int, C.c_int, vp, vp,
                                         C.c_size_t, vp]
    L.etree_kv_compact_paged.restype = C.c_int
    L.etree_device_status.argtypes = [vp, vp, C.POINTER(i32)]
    L.etree_device_status.restype = C.c_int
    L.etree_selftest_timeout.argtypes = [vp, C.c_size_t, vp]
    L.etree_selftest_timeout.restype = C.c_int
    L.etree_strerror.argtypes = [C.c_int]
    L.etree_strerror.restype = C.c_char_p
    L.etree_last_error.argtypes = []
    L.etree_last_error.restype = C.c_char_p
    L.etree_version.argtypes = []
    L.etree_version.restype = C.c_int
    L.etree_verify_attn_noalloc.argtypes = [bp, vp, vp, vp, vp, vp, i64, C.c_int, C.c_int,
                                            C.c_int, f32, vp, vp, vp, vp]
    L.etree_verify_attn_noalloc.restype = C.c_int
    ip = C.POINTER(C.c_int32)
    L.etree_attn_plan.argtypes = [bp, C.c_int, C.c_int, ip, ip, ip, ip, ip, ip]
    L.etree_attn_plan.restype = C.c_int
    _lib = L
    return L


def _check(st: int) -> int:
    if st != 0:
        raise EtreeError(st, lib().etree_last_error().decode())
    return st


def _ptr(t: torch.Tensor | None, dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def etree_lowrank_workspace_size(M: int, hidden_dim: int, rank: int, vocab: int) -> int:
    return int(lib().etree_lowrank_workspace_size(int(M), int(hidden_dim), int(rank),
                                                  int(vocab)))


def etree_lowrank_candidates(hidden, D, U, W, k: int, out_ids, out_logit, workspace,
                             stream=None, check: bool = True) -> int:
    """hidden [M, H], D [r, H], U [V, r], W [V, H] bf16; out_ids int32 / out_logit fp32 [M, k]."""
    bf = torch.bfloat16
    M, H = hidden.shape
    r, V = D.shape[0], U.shape[0]
    st = lib().etree_lowrank_candidates(
        _ptr(hidden, bf, "hidden"), M, H, _ptr(D, bf, "D"), _ptr(U, bf, "U"), r,
        _ptr(W, bf, "W"), V, int(k), _ptr(out_ids, torch.int32, "out_ids"),
        _ptr(out_logit, torch.float32, "out_logit"), _ptr(workspace, torch.uint8, "workspace"),
        workspace.numel(), _stream(stream))
    return _check(st) if check else st


class CostTable(C.Structure):
    _fields_ = [("nB", C.c_int32), ("nN", C.c_int32), ("nL", C.c_int32),
                ("B", C.POINTER(C.c_int32)), ("N", C.POINTER(C.c_int32)),
                ("L", C.POINTER(C.c_int32)), ("us", C.POINTER(C.c_float))]


class TreePlan(C.Structure):
    _fields_ = [("depth", C.c_int32), ("width", C.c_int32), ("nodes", C.c_int32),
                ("expected_accept", C.c_double), ("step_us", C.c_double),
                ("tokens_per_s", C.c_double)]


def cost_table(d: dict) -> CostTable:
    """An etree_cost_table over the dict {"B", "N", "L", "us"} (as calibrate.py writes it)."""
    import numpy as np
    arrs = [np.ascontiguousarray(d[k], dtype=np.int32) for k in ("B", "N", "L")]
    us = np.ascontiguousarray(d["us"], dtype=np.float32)
    if us.shape != (len(arrs[0]), len(arrs[1]), len(arrs[2])):
        raise ValueError(f"us has shape {us.shape}, want (|B|, |N|, |L|)")
    i32p, f32p = C.POINTER(C.c_int32), C.POINTER(C.c_float)
    t = CostTable(len(arrs[0]), len(arrs[1]), len(arrs[2]), arrs[0].ctypes.data_as(i32p),
                  arrs[1].ctypes.data_as(i32p), arrs[2].ctypes.data_as(i32p),
                  us.ctypes.data_as(f32p))
    t._keep = (arrs, us)
    return t


def load_cost_table(name: str = "b200_dense27b") -> dict:
    """A packaged calibration (cost_tables/<name>.json) or a path to one."""
    import json
    path = name if os.path.exists(name) else os.path.join(HERE, "cost_tables", name + ".json")
    with open(path) as f:
        return json.load(f)


def etree_verify_cost(table, B: float, N: float, L: float) -> float:
    t = table if isinstance(table, CostTable) else cost_table(table)
    out = C.c_double()
    _check(lib().etree_verify_cost(C.byref(t), float(B), float(N), float(L), C.byref(out)))
    return out.value


def etree_plan_tree(table, B: int, L: int, acc_rank, draft_us_per_level: float,
                    draft_us_fixed: float = 0.0, max_depth: int = 16, max_width: int = 16,
                    max_nodes: int = 64) -> dict:
    """The static (depth, width) draft tree with the most expected tokens/s (host only)."""
    t = table if isinstance(table, CostTable) else cost_table(table)
    acc = (C.c_float * len(acc_rank))(*[float(a) for a in acc_rank])
    out = TreePlan()
    _check(lib().etree_plan_tree(C.byref(t), int(B), int(L), acc, len(acc_rank),
                                 float(draft_us_per_level), float(draft_us_fixed),
                                 int(max_depth), int(max_width), int(max_nodes), C.byref(out)))
    return {k: getattr(out, k) for k, _ in TreePlan._fields_}


def make_batch(cu_nodes, parent, tokens, kv_len, slot_base, slot_cap, n_max: int,
               kv_len_max: int) -> Batch:
    """Wrap device int tensors as an etree_batch (keeps references to them)."""
    b = Batch()
    b.B = cu_nodes.numel() - 1
    b.n_total = parent.numel()
    b.n_max = int(n_max)
    b.kv_len_max = int(kv_len_max)
    b.cu_nodes = _ptr(cu_nodes, torch.int32, "cu_nodes")
    b.parent = _ptr(parent, torch.int32, "parent")
    b.tokens = _ptr(tokens, torch.int32, "tokens")
    b.kv_len = _ptr(kv_len, torch.int32, "kv_len")
    b.slot_base = _ptr(slot_base, torch.int64, "slot_base")
    b.slot_cap = _ptr(slot_cap, torch.int32, "slot_cap")
    b._keep = (cu_nodes, parent, tokens, kv_len, slot_base, slot_cap)
    return b


def etree_version() -> int:
    return int(lib().etree_version())


def etree_strerror(status: int) -> str:
    return lib().etree_strerror(int(status)).decode()


def etree_workspace_size(batch: Batch, hq: int, hkv: int, head_dim: int, hidden_dim: int,
                         vocab: int) -> int:
    return int(lib().etree_workspace_size(C.byref(batch), hq, hkv, head_dim, hidden_dim, vocab))


def etree_workspace_init(workspace: torch.Tensor, stream=None) -> None:
    _check(lib().etree_workspace_init(_ptr(workspace, torch.uint8, "workspace"),
                                      workspace.numel(), _stream(stream)))


def etree_verify_attn(batch: Batch, q, k_tree, v_tree, k_cache, v_cache, scale: float, out,
                      lse, workspace, stream=None, check: bool = True) -> int:
    bf = torch.bfloat16
    hq, d = q.shape[1], q.shape[2]
    hkv = k_tree.shape[1]
    st = lib().etree_verify_attn(
        C.byref(batch), _ptr(q, bf, "q"), _ptr(k_tree, bf, "k_tree"), _ptr(v_tree, bf, "v_tree"),
        _ptr(k_cache, bf, "k_cache"), _ptr(v_cache, bf, "v_cache"), k_cache.shape[0], hq, hkv,
        d, float(scale), _ptr(out, bf, "out"), _ptr(lse, torch.float32, "lse"),
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream))
    return _check(st) if check else st


def etree_verify_attn_noalloc(batch: Batch, q, k_tree, v_tree, k_cache, v_cache, scale: float,
                              out, lse, status_out=None, stream=None, check: bool = True) -> int:
    """Tree attention backed by the library's static scratch array: for callers that cannot
    allocate device memory (no workspace argument; see etree.h for the contract)."""
    bf = torch.bfloat16
    hq, d = q.shape[1], q.shape[2]
    hkv = k_tree.shape[1]
    st = lib().etree_verify_attn_noalloc(
        C.byref(batch), _ptr(q, bf, "q"), _ptr(k_tree, bf, "k_tree"), _ptr(v_tree, bf, "v_tree"),
        _ptr(k_cache, bf, "k_cache"), _ptr(v_cache, bf, "v_cache"), k_cache.shape[0], hq, hkv,
        d, float(scale), _ptr(out, bf, "out"), _ptr(lse, torch.float32, "lse"),
        _ptr(status_out, torch.int32, "status_out"), _stream(stream))
    return _check(st) if check else st


def etree_lmhead_accept(batch: Batch, hidden, w_lm, temperature: float, q_draft, seed: int,
                        step: int, accept_len, path, out_tokens, node_argmax, node_gap,
                        workspace, stream=None, check: bool = True) -> int:
    bf = torch.bfloat16
    st = lib().etree_lmhead_accept(
        C.byref(batch), _ptr(hidden, bf, "hidden"), _ptr(w_lm, bf, "w_lm"), hidden.shape[1],
        w_lm.shape[0], float(temperature), _ptr(q_draft, torch.float32, "q_draft"),
        int(seed) & (2**64 - 1), int(step) & (2**64 - 1),
        _ptr(accept_len, torch.int32, "accept_len"), _ptr(path, torch.int32, "path"),
        _ptr(out_tokens, torch.int32, "out_tokens"),
        _ptr(node_argmax, torch.int32, "node_argmax"), _ptr(node_gap, torch.float32, "node_gap"),
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream))
    return _check(st) if check else st


def etree_lmhead_accept_tree(batch: Batch, hidden, w_lm, temperature: float, q_draft, seed: int,
                             step: int, accept_len, path, out_tokens, zbuf, workspace,
                             stream=None, check: bool = True) -> int:
    """zbuf: fp32 [rows][vocab] device tensor (or None for no rows)."""
    bf = torch.bfloat16
    rows = 0 if zbuf is None else int(zbuf.shape[0])
    st = lib().etree_lmhead_accept_tree(
        C.byref(batch), _ptr(hidden, bf, "hidden"), _ptr(w_lm, bf, "w_lm"), hidden.shape[1],
        w_lm.shape[0], float(temperature), _ptr(q_draft, torch.float32, "q_draft"),
        int(seed) & (2**64 - 1), int(step) & (2**64 - 1),
        _ptr(accept_len, torch.int32, "accept_len"), _ptr(path, torch.int32, "path"),
        _ptr(out_tokens, torch.int32, "out_tokens"), _ptr(zbuf, torch.float32, "zbuf"), rows,
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream))
    return _check(st) if check else st


def etree_lmhead_accept_timed(batch: Batch, hidden, w_lm, temperature: float, q_draft, seed: int,
                              step: int, accept_len, path, out_tokens, node_argmax, node_gap,
                              zbuf, branching: bool, marks, workspace, stream=None,
                              check: bool = True) -> int:
    """etree_lmhead_accept(_tree) with phase marks: `marks` is a list of 4 torch.cuda.Event
    (or None entries) recorded after the set-up kernels, the first GEMM, the acceptance kernels
    and the draw GEMM.  torch creates an Event's CUDA event on its first record(): record each
    once before passing it, or its handle is NULL and the mark is skipped."""
    bf = torch.bfloat16
    rows = 0 if zbuf is None else int(zbuf.shape[0])
    arr = (C.c_void_p * 4)(*[None if m is None else m.cuda_event for m in marks])
    st = lib().etree_lmhead_accept_timed(
        C.byref(batch), _ptr(hidden, bf, "hidden"), _ptr(w_lm, bf, "w_lm"), hidden.shape[1],
        w_lm.shape[0], float(temperature), _ptr(q_draft, torch.float32, "q_draft"),
        int(seed) & (2**64 - 1), int(step) & (2**64 - 1),
        _ptr(accept_len, torch.int32, "accept_len"), _ptr(path, torch.int32, "path"),
        _ptr(out_tokens, torch.int32, "out_tokens"),
        _ptr(node_argmax, torch.int32, "node_argmax"), _ptr(node_gap, torch.float32, "node_gap"),
        _ptr(zbuf, torch.float32, "zbuf"), rows, int(bool(branching)), arr,
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream))
    return _check(st) if check else st


def etree_verify_attn_paged(batch: Batch, block_table, page_size: int, q, k_tree, v_tree,
                            k_pool, v_pool, scale: float, out, lse, workspace, stream=None,
                            check: bool = True) -> int:
    """block_table: int32 [B, max_pages] device tensor; pools [num_pages * page_size, hkv, d]."""
    bf = torch.bfloat16
    hq, d = q.shape[1], q.shape[2]
    hkv = k_tree.shape[1]
    num_pages = k_pool.shape[0] // int(page_size)
    st = lib().etree_verify_attn_paged(
        C.byref(batch), _ptr(block_table, torch.int32, "block_table"), block_table.shape[1],
        int(page_size), _ptr(q, bf, "q"), _ptr(k_tree, bf, "k_tree"), _ptr(v_tree, bf, "v_tree"),
        _ptr(k_pool, bf, "k_pool"), _ptr(v_pool, bf, "v_pool"), num_pages, hq, hkv, d,
        float(scale), _ptr(out, bf, "out"), _ptr(lse, torch.float32, "lse"),
        _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream))
    return _check(st) if check else st


def _check_path(batch: Batch, path):
    # the library reads a full row of ETREE_PATH_STRIDE entries per request
    if isinstance(path, torch.Tensor) and path.numel() < batch.B * 64:
        raise ValueError(f"path must hold [B][64] entries, got {tuple(path.shape)}")


def etree_kv_compact_paged(batch: Batch, block_table, page_size: int, accept_len, path, k_tree,
                           v_tree, k_pool, v_pool, num_pages: int, n_layers: int,
                           tree_layer_stride: int, cache_layer_stride: int, kv_len_out,
                           workspace, stream=None, check: bool = True) -> int:
    bf = torch.bfloat16
    _check_path(batch, path)
    hkv, d = k_tree.shape[-2], k_tree.shape[-1]
    st = lib().etree_kv_compact_paged(
        C.byref(batch), _ptr(block_table, torch.int32, "block_table"), block_table.shape[1],
        int(page_size), _ptr(accept_len, torch.int32, "accept_len"),
        _ptr(path, torch.int32, "path"), _ptr(k_tree, bf, "k_tree"), _ptr(v_tree, bf, "v_tree"),
        _ptr(k_pool, bf, "k_pool"), _ptr(v_pool, bf, "v_pool"), int(num_pages), int(n_layers),
        int(tree_layer_stride), int(cache_layer_stride), hkv, d,
        _ptr(kv_len_out, torch.int32, "kv_len_out"), _ptr(workspace, torch.uint8, "workspace"),
        workspace.numel(), _stream(stream))
    return _check(st) if check else st


def etree_kv_compact(batch: Batch, accept_len, path, k_tree, v_tree, k_cache, v_cache,
                     n_layers: int, tree_layer_stride: int, cache_layer_stride: int, kv_len_out,
                     workspace, stream=None, check: bool = True) -> int:
    bf = torch.bfloat16
    _check_path(batch, path)
    hkv, d = k_tree.shape[-2], k_tree.shape[-1]
    st = lib().etree_kv_compact(
        C.byref(batch), _ptr(accept_len, torch.int32, "accept_len"),
        _ptr(path, torch.int32, "path"), _ptr(k_tree, bf, "k_tree"), _ptr(v_tree, bf, "v_tree"),
        _ptr(k_cache, bf, "k_cache"), _ptr(v_cache, bf, "v_cache"), int(n_layers),
        int(tree_layer_stride), int(cache_layer_stride), hkv, d,
        _ptr(kv_len_out, torch.int32, "kv_len_out"), _ptr(workspace, torch.uint8, "workspace"),
        workspace.numel(), _stream(stream))
    return _check(st) if check else st


def etree_attn_plan(batch: Batch, hq: int, hkv: int) -> dict:
    v = [C.c_int32(0) for _ in range(6)]
    _check(lib().etree_attn_plan(C.byref(batch), hq, hkv, *[C.byref(x) for x in v]))
    return dict(zip(["kernel", "rows_per_cta", "row_blocks", "splits", "tiles_per_split",
                     "launches"], [int(x.value) for x in v]))


def etree_selftest_timeout(workspace: torch.Tensor, stream=None, check: bool = True) -> int:
    """Enqueue the bounded-wait self-test; etree_device_status then reports ETREE_ETIMEOUT."""
    st = lib().etree_selftest_timeout(_ptr(workspace, torch.uint8, "workspace"),
                                      workspace.numel(), _stream(stream))
    return _check(st) if check else st


def etree_device_status(workspace: torch.Tensor, stream=None) -> tuple[int, int]:
    det = C.c_int32(0)
    st = lib().etree_device_status(_ptr(workspace, torch.uint8, "workspace"), _stream(stream),
                                   C.byref(det))
    return int(st), int(det.value)
