"""Host logic of the benchmark's roofline entry: the DRAM traffic recorded in a
profile summary is reported only while the kernel's sources are the ones the
capture ran on, and every committed summary the benchmark reads parses."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _write_profile(root, tag, workload, source_hash, traffic):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    with open(os.path.join(root, "profiles", f"{tag}__{workload}.md"), "w") as f:
        f.write(f"# {tag}\n\n- source_hash: {source_hash}\n- traffic_bytes_per_launch: {traffic}\n")


def _copy_sources(tmp_path):
    import shutil
    src = os.path.join(ROOT, "gqa_decode_attention_kvattn_b200", "csrc")
    dst = os.path.join(str(tmp_path), "gqa_decode_attention_kvattn_b200", "csrc")
    shutil.copytree(src, dst)
    return dst


def test_traffic_reported_only_for_matching_sources(tmp_path, monkeypatch):
    _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    tag = "prefill_chunk"
    current = bench.kernel_source_hash(tag)
    _write_profile(str(tmp_path), tag, "w_match", current, 123456789)
    _write_profile(str(tmp_path), tag, "w_stale", "0" * 16, 123456789)
    assert bench.profiled_traffic(tag, "w_match") == 123456789.0
    assert bench.profiled_traffic(tag, "w_stale") is None   # the kernel changed since
    assert bench.profiled_traffic(tag, "w_missing") is None  # no capture at all


def test_source_hash_follows_every_listed_file(tmp_path, monkeypatch):
    # an edit to any file a kernel is built from changes that kernel's hash
    dst = _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    for tag, files in bench.KERNEL_SOURCES.items():
        before = bench.kernel_source_hash(tag)
        assert len(before) == 16 and bench.kernel_source_hash(tag) == before
        for name in files:
            path = os.path.join(dst, name)
            with open(path, "rb") as f:
                orig = f.read()
            with open(path, "ab") as f:
                f.write(b"\n// edited\n")
            assert bench.kernel_source_hash(tag) != before, (tag, name)
            with open(path, "wb") as f:
                f.write(orig)
        assert bench.kernel_source_hash(tag) == before


def test_committed_profiles_parse():
    # every summary the benchmark reads names the source hash its capture ran
    # on and a positive per-launch DRAM traffic (a kernel edited since the
    # capture makes the benchmark report null traffic, not a wrong number)
    import re
    for tag, workload in (("decode_mma", "decode_ragged_b64_l32"),
                          ("decode_tc", "decode_mqa_g32_b64"),
                          ("prefill_chunk", "prefill_b4_t512_sp3584")):
        with open(os.path.join(ROOT, "profiles", f"{tag}__{workload}.md")) as f:
            text = f.read()
        assert re.search(r"^- source_hash: [0-9a-f]{16}$", text, re.M), (tag, workload)
        m = re.search(r"^- traffic_bytes_per_launch: ([0-9]+)$", text, re.M)
        assert m and int(m.group(1)) > 0, (tag, workload)
