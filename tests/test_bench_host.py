"""Host-side pieces of bench.py that need no GPU: the digest that ties a committed ncu
capture to the kernel code it was taken on, the committed traffic records, and the bounded
oracle samples of the CPU baseline and the reference arm."""
import importlib.util
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test",
                                                  os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def test_digest_ignores_comments_and_layout_but_not_code(bench, tmp_path, monkeypatch):
    csrc = tmp_path / "block_sparse_paged_scores_b200" / "csrc"
    csrc.mkdir(parents=True)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (csrc / "k.cu").write_text("int f(int a) { return a + 1; }  // one\n")
    d0 = bench.source_digest("k.cu")
    (csrc / "k.cu").write_text("/* two */\nint f(int a) {\n  return a + 1;\n}\n")
    assert bench.source_digest("k.cu") == d0
    (csrc / "k.cu").write_text("int f(int a) { return a + 2; }\n")
    assert bench.source_digest("k.cu") != d0


def test_traffic_records_are_complete(bench):
    d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    known = set(bench.VARIANTS) | {"bf16_decode", "ragged_prefill", "spec_decode",
                                   "fp8_long_decode", "tiny_decode"}
    for key, e in d.items():
        kernel, workload = key.split("/")
        assert kernel in ("index_scores", "attention") and workload in known
        assert e["dram_bytes_per_launch"] > 0 and e["captured_dram_bytes_per_launch"] > 0
        assert "captured_workload" in e and "source_digest" in e
    # the headline's dominant kernel (the indexer on FP8 long-context decode) and the attention
    # kernels have committed captures of their current code
    index = bench.source_digest("indexer.cu", "select_row.cuh")
    for w in ("fp8_long_decode", "fp8_long_decode_fp8_index_k", "fp8_long_decode_fp4_index_k"):
        assert bench.profiled_traffic("index_scores", w, index) is not None, w
    stream = bench.source_digest("attention_stream.cu", "attn_common.cuh", "select_row.cuh")
    for w in ("bf16_decode", "spec_decode", "spec_decode_shared_topk"):
        assert bench.profiled_traffic("attention", w, stream) is not None, w
    assert bench.profiled_traffic("attention", "ragged_prefill",
                                  bench.source_digest("attention_tc.cu")) is not None
    assert bench.profiled_traffic("attention", "bf16_decode", "0" * 16) is None


@pytest.mark.parametrize("workload", ["tiny_decode", "bf16_decode", "spec_decode",
                                      "fp8_long_decode", "ragged_prefill",
                                      "spec_decode_shared_topk", "fp8_long_decode_fp4_index_k",
                                      "ragged_prefill_fp8_kv"])
def test_oracle_samples_are_bounded(bench, workload):
    p, desc, share = bench.oracle_sample(workload, 4, seed=7)
    assert share == (workload == "spec_decode_shared_topk")
    base, changes, _ = bench.VARIANTS.get(workload, (workload, {}, {}))
    if "idx_dtype" in changes:
        assert p["idx_dtype"] == changes["idx_dtype"]
    if "kv_dtype" in changes:
        assert p["kv_fp8"]
    assert p["batch"] <= 4
    if p["max_q_len"] > 8:           # prefill: one sequence with 16-64 new tokens
        assert p["batch"] == 1 and 16 <= p["total_q"] <= 64
    else:
        assert p["total_q"] <= 4 * 8
    assert workload in desc
