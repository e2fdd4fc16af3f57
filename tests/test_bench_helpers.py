"""Host-side parts of bench.py (no GPU): the source fingerprint that ties a committed ncu traffic
figure to the kernel sources it was measured on, the packed step-input buffer, and the oracle
(reference) arm's JSON line."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_strip_comments_keeps_code_and_literals():
    src = ('int a = 1; // trailing\n'
           '/* block\n comment */ float b = 2.f;\n'
           'const char* s = "not // a comment";\n'
           "char c = '/';  char d = '\\'';\n"
           '  int   e  =  3 ;')
    out = bench.strip_comments(src)
    assert "trailing" not in out and "block" not in out
    assert '"not // a comment"' in out
    assert "'/'" in out and "'\\''" in out
    assert "int a = 1;" in out and "float b = 2.f;" in out and "int e = 3 ;" in out


def test_comment_edits_do_not_change_the_fingerprint(tmp_path, monkeypatch):
    csrc = tmp_path / "draft_tree_verification_masked_b200" / "csrc"
    csrc.mkdir(parents=True)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (csrc / "k.cu").write_text("// v1\n__global__ void k(int* p) { p[0] = 1; }\n")
    h1 = bench.source_hash("k.cu")
    (csrc / "k.cu").write_text("/* a new comment */\n__global__  void k(int* p) {\n  p[0] = 1; }\n")
    assert bench.source_hash("k.cu") == h1
    (csrc / "k.cu").write_text("__global__ void k(int* p) { p[0] = 2; }\n")
    assert bench.source_hash("k.cu") != h1



def test_packed_buffer_layout():
    """The step's inputs share one buffer: every tensor starts on a 256-byte boundary, none
    overlaps the next, and the views alias the buffer (a copy into the buffer reaches them)."""
    import torch
    from draft_tree_verification_masked_b200.runner import Packed
    specs = [("a", (5,), torch.int32), ("b", (3, 7), torch.int64), ("c", (2, 3, 4), torch.bfloat16),
             ("d", (1,), torch.float32)]
    pk = Packed(specs, "cpu")
    prev_end = 0
    for name, shape, dtype in specs:
        off = pk.offset(name)
        v = pk.view(name)
        assert off % 256 == 0 and off >= prev_end, name
        assert tuple(v.shape) == shape and v.dtype == dtype, name
        prev_end = off + v.numel() * v.element_size()
    assert pk.buf.numel() >= prev_end
    pk.buf.copy_(torch.arange(pk.buf.numel(), dtype=torch.int64).to(torch.uint8))
    a = pk.view("a")
    assert bytes(a.numpy().tobytes()) == bytes(pk.buf[:20].numpy().tobytes())
    # the tail from a tensor's offset holds it and everything after it
    tail = pk.buf[pk.offset("c"):]
    assert tail.numel() >= pk.view("c").numel() * 2 + pk.view("d").numel() * 4


def _reference_arm(env_extra):
    import json
    import subprocess
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "tiny", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return [json.loads(ln) for ln in lines]


def test_reference_arm_prints_one_contract_line():
    """The oracle arm runs on host cores only: one JSON line with the main arm's metric, unit and
    workload keys, an oracle cpu_baseline and an e2e block that moves no bytes."""
    from draft_tree_verification_masked_b200 import workload as W
    (line,) = _reference_arm({"RANK": "0", "WORLD_SIZE": "1"})
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "accepted tok/s" and line["higher_is_better"] is True
    assert line["steps"] == 1 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["value"] > 0 and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    want = bench.workload_config("tiny", W.generate("tiny"), 1)
    assert {k: line["config"][k] for k in want} == want


def test_reference_arm_runs_on_rank_zero_only():
    assert _reference_arm({"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_algorithmic_work_matches_the_per_unit_figures():
    """The roofline numerators: attention reads the KV cache once (2 L Hkv D 2 bytes) plus the
    tree K/V, Q and O, and does 4 Hq D FLOPs per (query node, visible key); the LM head reads W
    once and does 2 N V H FLOPs; compaction reads and writes (a + 1) K and V rows per layer."""
    from types import SimpleNamespace

    import numpy as np
    from draft_tree_verification_masked_b200 import workload as W

    wl = W.generate("dense27b_b1", hidden=64, vocab=256)
    L, Hkv, Hq, D, N = 4096, 8, 40, 128, 64
    b, f = bench.attn_work(wl)
    assert b == 2 * L * Hkv * D * 2 + 2 * N * Hkv * D * 2 + 2 * N * Hq * D * 2
    # visible tree keys = sum over nodes of their subtree sizes (pairs ancestor-or-self, node)
    size = np.ones(N, dtype=np.int64)
    for i in range(N - 1, 0, -1):
        size[wl.parent[i]] += size[i]
    assert f == 4 * Hq * D * (N * L + int(size.sum()))
    assert abs(f / 5.37e9 - 1) < 0.01                         # 5.37 GFLOP at this shape
    head = SimpleNamespace(vocab=151936, hidden_dim=5120, n_total=64)
    hb, hf = bench.lmhead_work(head)
    assert hb == 151936 * 5120 * 2 + 64 * 5120 * 2 and abs(hb / 1.556e9 - 1) < 0.001
    assert hf == 2 * 64 * 151936 * 5120
    kv = SimpleNamespace(hkv=8, head_dim=128)
    assert bench.compact_work(kv, np.array([3, 0])) == 2 * 2 * (4 + 1) * 8 * 128 * 2
    assert bench.compact_work(kv, np.array([3, 0]), n_layers=64) == 64 * 2 * 2 * 5 * 8 * 128 * 2
