"""The DRAM traffic the benchmark reports comes from a committed ncu summary,
and only while that summary was taken on the kernel's current source: a
changed kernel reports null until it is profiled again."""
import json
import os
import shutil

import bench


def write_traffic(root, entries):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    with open(os.path.join(root, "profiles", "traffic.json"), "w") as f:
        json.dump(entries, f)


def test_traffic_only_while_the_source_matches(tmp_path, monkeypatch):
    root = str(tmp_path)
    write_traffic(root, {"attn_partial.cu": {"dense_p16": {"dram_bytes_per_launch": 123.0,
                                                           "report": "x.md", "source_hash": "abc"}}})
    monkeypatch.setattr(bench, "ROOT", root)
    monkeypatch.setattr(bench, "kernel_source_hash", lambda name: "abc")
    assert bench.recorded_traffic("attn_partial.cu", "dense_p16") == 123.0
    assert bench.recorded_traffic("attn_partial.cu", "frame_tile_8x3600") is None
    assert bench.recorded_traffic("merge.cu", "dense_p16") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda name: "abd")
    assert bench.recorded_traffic("attn_partial.cu", "dense_p16") is None


def test_no_traffic_file_means_null(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("attn_partial.cu", "dense_p16") is None


def test_source_hash_covers_the_shared_header(tmp_path, monkeypatch):
    src = os.path.join(bench.ROOT, "sparse_state_reuse_b200", "csrc")
    dst = os.path.join(str(tmp_path), "sparse_state_reuse_b200", "csrc")
    shutil.copytree(src, dst, ignore=shutil.ignore_patterns("*.o", "*.so"))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    before = {k: bench.kernel_source_hash(k) for k in ("attn_partial.cu", "merge.cu")}
    with open(os.path.join(dst, "common.cuh"), "a") as f:
        f.write("\n// edited\n")
    after = {k: bench.kernel_source_hash(k) for k in ("attn_partial.cu", "merge.cu")}
    assert all(before[k] != after[k] for k in before)
    # the merge also hashes the weights header it shares with the plan
    with open(os.path.join(dst, "weights.cuh"), "a") as f:
        f.write("\n// edited\n")
    assert bench.kernel_source_hash("merge.cu") != after["merge.cu"]
    assert bench.kernel_source_hash("attn_partial.cu") == after["attn_partial.cu"]


def test_committed_entries_name_their_summaries():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    assert d
    for kernel, entries in d.items():
        for workload, e in entries.items():
            assert e["dram_bytes_per_launch"] > 0, (kernel, workload)
            assert len(e["source_hash"]) == 16, (kernel, workload)
            report = os.path.join(bench.ROOT, "profiles", e["report"])
            assert os.path.exists(report), report
            with open(report) as f:
                text = f.read()
            assert e["source_hash"] in text and "--clock-control none" in text, report
