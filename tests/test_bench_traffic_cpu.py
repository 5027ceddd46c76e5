"""bench.py's roofline traffic: DRAM bytes per launch come from the committed
ncu record only when the record was taken on the current decode-kernel source
(the record is keyed by a hash of it); otherwise the line carries null."""
import json
import os
import shutil

import bench


def _tree(tmp_path):
    src = os.path.join(bench.ROOT, "paged_kv_cache_340_b200", "csrc")
    dst = tmp_path / "paged_kv_cache_340_b200" / "csrc"
    dst.mkdir(parents=True)
    for name in ("pa_decode.cu", "pa_common.cuh", "pa_internal.h"):
        shutil.copy(os.path.join(src, name), dst / name)
    (tmp_path / "profiles").mkdir()
    return tmp_path


def test_recorded_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    root = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    sha = bench.kernel_source_sha()
    assert len(sha) == 16
    rec = {"w": {"k": {"source_sha": sha, "dram_bytes_per_launch": 1234}}}
    (root / "profiles" / "decode_dram_traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("w", "k") == 1234
    assert bench.recorded_traffic("w", "other") is None   # another kernel
    assert bench.recorded_traffic("x", "k") is None       # another workload
    # any edit of the decode source (a comment too) makes the record stale
    f = root / "paged_kv_cache_340_b200" / "csrc" / "pa_common.cuh"
    f.write_text(f.read_text() + "\n// edited\n")
    assert bench.kernel_source_sha() != sha
    assert bench.recorded_traffic("w", "k") is None


def test_recorded_traffic_without_a_record(tmp_path, monkeypatch):
    root = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.recorded_traffic("w", "k") is None


def test_committed_record_is_well_formed():
    """Every entry of the committed record names its source hash, its bytes
    (read + write) and the command that took them."""
    with open(os.path.join(bench.ROOT, "profiles", "decode_dram_traffic.json")) as f:
        rec = json.load(f)
    assert rec
    for workload, kernels in rec.items():
        for kernel, e in kernels.items():
            assert len(e["source_sha"]) == 16
            assert abs(e["dram_bytes_per_launch"] - e["dram_bytes_read"] - e["dram_bytes_write"]) <= 1
            assert e["dram_bytes_per_launch"] > 0
            assert "--clock-control none" in e["command"] and f"--workload {workload}" in e["command"]
