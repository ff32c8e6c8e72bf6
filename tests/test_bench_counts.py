"""The algorithmic work bench.py divides by (the numerators of every reported
roofline fraction), checked against row-by-row counts on small shapes, and
the rule that a recorded ncu traffic figure is dropped once its kernel's
sources change.

Counts (HiLS paper, aitrends.kr article, sections "방법론" and "기술 상세"):
each row scores every candidate chunk (the chunks before its local window)
with one d-long dot product (2d FLOPs); it attends min(K, candidates) chunks
of C keys plus its window's keys up to itself, each key costing a d-long
logit and a d-long value update (4d FLOPs).  A decode step reads, per
(sequence, kv head), the union of its query heads' kept chunks plus the
window's chunks: 64 key rows and 64 value rows of d elements each.
"""
import numpy as np
import pytest

import bench
from chunk_wise_sparse_b200.inputs import custom


def row_by_row(w):
    wc = max(1, w.window // w.C)
    score = attn = 0
    for i in range(w.N):
        own = i // w.C
        n_cand = max(0, own - (wc - 1))
        first_window_key = n_cand * w.C
        score += n_cand
        attn += min(w.K, n_cand) * w.C + (i - first_window_key + 1)
    rows = w.B * w.Hq
    return 2 * w.d * rows * score, 4 * w.d * rows * attn


@pytest.mark.parametrize("N,K,window", [(1024, 3, 0), (1024, 3, 256), (4288, 16, 0), (2048, 64, 512),
                                        (640, 1, 640)])
def test_useful_flops_match_a_row_by_row_count(N, K, window):
    w = custom("count", B=2, Hq=4, Hkv=2, d=64, N=N, K=K, window=window)
    score, attn = row_by_row(w)
    u = bench.useful_work(w)
    assert u["flops_score"] == score
    assert u["flops_attn"] == attn


def test_decode_selected_bytes_is_the_union_per_kv_head():
    rng = np.random.default_rng(5)
    for window, dtype in [(0, "bf16"), (512, "bf16"), (0, "fp32")]:
        w = custom("dec", B=3, Hq=8, Hkv=2, d=128, N=8192, K=6, window=window, dtype=dtype, kind="decode")
        nc = w.N // w.C
        ids = rng.integers(0, nc // 4, size=(w.B, w.Hq, w.K)).astype(np.int32)   # many shared chunks
        ids[0, 0, -2:] = -1                                                     # padding
        n_win = min(max(1, w.window // w.C), nc)
        elem = 2 if dtype == "bf16" else 4
        want = 0
        for b in range(w.B):
            for h in range(w.Hkv):
                chunks = set()
                for g in range(w.G):
                    chunks |= {int(c) for c in ids[b, h * w.G + g] if c >= 0}
                want += (len(chunks) + n_win) * w.C * w.d * elem * 2
        assert bench.decode_selected_bytes(ids, w) == want


def test_recorded_traffic_needs_the_sources_it_was_taken_on(monkeypatch, tmp_path):
    """A record applies only while the hash of its kernel's code is the one it
    was taken with (a temporary record, so the test does not depend on the
    committed one)."""
    import json
    (tmp_path / "profiles").mkdir()
    rec = {"per_row_bytes": {"select": 160.0},
           "per_step_bytes": {"decode:decode-128k-b8-gqa4-d128": 3.0e8},
           "sources_sha256": {"select": "h-select", "decode": "h-decode"}}
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernels_sha256", lambda kernel: "h-" + kernel)
    assert bench.recorded_traffic("select", 10) == pytest.approx(1600.0)
    assert bench.recorded_step_traffic("decode", "decode-128k-b8-gqa4-d128") == pytest.approx(3.0e8)
    assert bench.recorded_step_traffic("decode", "some-other-workload") is None
    monkeypatch.setattr(bench, "kernels_sha256", lambda kernel: "changed")
    assert bench.recorded_traffic("select", 10) is None
    assert bench.recorded_step_traffic("decode", "decode-128k-b8-gqa4-d128") is None


def test_source_hash_sees_code_not_comments():
    a = "int x = 1;  // a note\n/* a block\n   comment */ int y = 2;\n"
    b = "int x = 1;\nint y = 2;  // another note\n"
    assert bench.code_only(a) == bench.code_only(b)
    assert bench.code_only(a) != bench.code_only(a.replace("2", "3"))


def test_decode_cpu_baseline_times_the_oracle_decode_step():
    from chunk_wise_sparse_b200.inputs import generate
    for window in (0, 256):
        w = custom("dec-cpu", B=3, Hq=4, Hkv=2, d=64, N=2048, K=4, window=window, kind="decode")
        us, desc, threads = bench.cpu_oracle_decode(w, generate(w), budget_s=0.05)
        assert us > 0 and threads >= 1
        assert "1 of 3 sequences" in desc


def test_backward_cpu_baseline_times_one_slab_of_the_oracle_backward():
    from chunk_wise_sparse_b200.inputs import generate
    for window, Hq in ((0, 4), (192, 2)):
        w = custom("bwd-cpu", B=2, Hq=Hq, Hkv=2, d=64, N=512, K=3, window=window, dtype="fp32")
        v, desc, threads = bench.cpu_oracle_backward(w, generate(w))
        assert v > 0 and threads >= 1
        assert "1 of 4 (b, kv head) slabs" in desc
