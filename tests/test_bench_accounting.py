"""The roofline accounting of bench.py, checked on the CPU.

The algorithmic bytes of a decode step are the page bounds of every page, the
codes of the kept pages' tokens, the gathered K and V rows of the selected
tokens, R and W, the queries and outputs, and the index outputs; here they
are recomputed from the layout sizes of the 128K workload.  The profile hash
must ignore comments but not code.
"""
import os
import shutil

import bench
from workloads import get


def test_algorithmic_bytes_of_the_128k_step():
    w = get("llama8b_128k")
    parts, total = bench.algorithmic_bytes(w, w.N, w.P, w.k)
    units = w.B * w.Hkv                               # 8 (sequence, KV head) pairs
    pages = w.N // w.page                             # 8192 pages of 16 tokens
    assert parts["meta"] == units * pages * 2 * 128 * 2          # bf16 lower + upper bound rows
    assert parts["codes"] == units * w.P * w.page * (w.bits // 8)  # 512 kept pages x 16 tokens x 16 B
    assert parts["kv"] == units * w.k * 2 * 128 * 2              # 4096 K and V rows of 256 B
    assert parts["rw"] == w.Hkv * (128 * 128 + 128 * w.bits) * 4
    assert total == sum(parts.values()) == 52_600_864
    # at the measured copy bandwidth of this machine (6525.2 GB/s) this is 8.06 us
    assert abs(total / 6525.2e9 * 1e6 - 8.061) < 0.01


def test_budgets_larger_than_the_context_keep_everything():
    w = get("tiny_4k")
    parts, _ = bench.algorithmic_bytes(w, 100, 10_000, 10_000)
    assert parts["codes"] == w.B * w.Hkv * 100 * (w.bits // 8)   # every valid token is a candidate
    assert parts["kv"] == w.B * w.Hkv * 100 * 2 * 128 * 2        # and every one is selected


def test_profile_hash_ignores_comments_only(tmp_path, monkeypatch):
    csrc = tmp_path / "kv_cache_retrieval_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("decode.cu", "hhr_internal.cuh"):
        shutil.copy(os.path.join(bench.ROOT, "kv_cache_retrieval_b200", "csrc", f), csrc / f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    with open(csrc / "decode.cu", "a") as fh:
        fh.write("\n// a comment\n\n")
    assert bench.kernel_source_hash() == h0
    with open(csrc / "decode.cu", "a") as fh:
        fh.write("static int unused_symbol_for_the_test;\n")
    assert bench.kernel_source_hash() != h0


def test_planted_recall_counts_selected_tokens_and_kept_pages():
    import numpy as np
    tok_idx = np.array([[[5, 17, 40, -1]]], np.int32)          # one unit, 3 selected
    n_sel = np.array([[3]], np.int32)
    page_idx = np.array([[[0, 2, -1]]], np.int32)               # pages of 16 tokens: 0..15, 32..47
    planted = np.array([[[5, 20, 40, 47]]], np.int64)
    r = bench.planted_recall(tok_idx, n_sel, page_idx, planted, 16)
    assert r == {"tokens": 0.5, "pages": 0.75, "planted": 4}   # 5, 40 selected; 20 on page 1 (dropped)
    assert bench.planted_recall(tok_idx, n_sel, page_idx, planted[:, :, :0], 16) is None
