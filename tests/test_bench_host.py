"""Host logic of bench.py that needs no GPU: the per-op DRAM-traffic lookup
(a stored ncu figure is reported only for the kernel sources and the shape
it was captured on) and the FLOP counts per admitted pair."""
import importlib.util
import json
import os
import sys

import pytest

ROOT = os.path.join(os.path.dirname(__file__), "..")


@pytest.fixture(scope="module")
def bench():
    sys.path.insert(0, ROOT)
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_kernel_hash_is_per_op_and_stable(bench):
    hashes = {op: bench.kernel_hash(op) for op in bench.KERNEL_SOURCES}
    assert len(set(hashes.values())) == len(hashes)
    assert all(bench.kernel_hash(op) == h for op, h in hashes.items())


def test_kernel_hash_ignores_comments_and_layout_only(bench):
    src = 'int f(int a) {  // first\n  return a + 1; /* "x" */\n}\nconst char* s = "// kept";\n'
    assert bench.code_only(src) == bench.code_only(
        'int f(int a) {\n    return a + 1;\n}  // other words\nconst char* s = "// kept";')
    assert bench.code_only(src) != bench.code_only(src.replace("a + 1", "a + 2"))
    assert bench.code_only(src) != bench.code_only(src.replace('"// kept"', '"// gone"'))


def test_stored_traffic_requires_matching_source_and_shape(bench, tmp_path, monkeypatch):
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps({
        "tf": {"kernel_hash": bench.kernel_hash("jvp"), "H": 12, "dram_bytes_per_launch": 123},
        "tf_bwd": {"kernel_hash": "0" * 16, "H": 12, "dram_bytes_per_launch": 456},
        "tf_cache": {"kernel_hash": bench.kernel_hash("cache"), "H": 12, "Lq": 1560, "Lk": 32760,
                     "dram_bytes_per_launch": 789},
    }))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.stored_traffic("tf", H=12) == 123
    assert bench.stored_traffic("tf", H=2) is None             # another head count
    assert bench.stored_traffic("tf_bwd", "bwd", H=12) is None  # captured on other sources
    assert bench.stored_traffic("tf_cache", "cache", H=12, Lq=1560, Lk=32760) == 789
    assert bench.stored_traffic("tf_cache", "cache", H=12, Lq=4680, Lk=32760) is None
    assert bench.stored_traffic("missing") is None


def test_committed_traffic_entries_name_their_capture(bench):
    with open(bench.TRAFFIC_FILE) as f:
        d = json.load(f)
    for key, e in d.items():
        assert e["dram_bytes_per_launch"] == e["dram_bytes_read"] + e["dram_bytes_write"], key
        assert os.path.exists(os.path.join(ROOT, e["source"])), key


def test_flops_per_pair(bench):
    class W:
        d = 128
    assert bench.flops_per_pair(W, "jvp") == 12 * 128
    assert bench.flops_per_pair(W, "bwd") == 10 * 128


def test_workload_label_names_its_own_mask(bench):
    from attention_jvp_continuous_b200.inputs import WORKLOADS
    labels = {n: bench.describe_workload(w) for n, w in WORKLOADS.items()}
    assert "frame-causal" in labels["frame_causal"] and "teacher" not in labels["frame_causal"]
    assert "clean,noisy" not in labels["frame_causal"]
    assert "chunks of 3 frames" in labels["chunk_tf"]
    assert "frame-wise teacher-forcing" in labels["tf"]
    assert "U(0.5, 2)" in labels["tf_long"] and "102960 tokens" in labels["tf_long"]
