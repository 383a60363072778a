"""The bench's DRAM-traffic record on CPU: a family's per-launch DRAM bytes are reported only
while the CUDA sources hash to the value the counters were taken with, and the record covers
every family the bench times."""
import json
import os
import re
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _fake_root(tmp_path, record):
    """A copy of the CUDA sources and a traffic record under tmp_path."""
    shutil.copytree(os.path.join(ROOT, "alibi_rope_tile_b200", "csrc"), tmp_path / "alibi_rope_tile_b200" / "csrc")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(record))
    return tmp_path


def test_traffic_is_reported_only_for_the_sources_it_was_taken_with(tmp_path, monkeypatch):
    root = _fake_root(tmp_path, {})
    monkeypatch.setattr(bench, "ROOT", str(root))
    record = {"csrc_sha256": bench.csrc_sha256(), "per_launch_dram_bytes": {"gqa_prefill": 123}}
    (root / "profiles" / "traffic.json").write_text(json.dumps(record))
    assert bench.measured_traffic() == {"gqa_prefill": 123}
    # one byte of one kernel source changes: the counters no longer describe the kernels
    src = root / "alibi_rope_tile_b200" / "csrc" / "gemm_tc.cu"
    src.write_bytes(src.read_bytes() + b"\n")
    assert bench.measured_traffic() == {}
    # no record at all
    (root / "profiles" / "traffic.json").unlink()
    assert bench.measured_traffic() == {}


def test_traffic_record_covers_every_timed_family():
    with open(os.path.join(ROOT, "bench.py")) as f:
        families = set(re.findall(r'want\("([a-z0-9_]+)"\)', f.read()))
    assert {"gqa_prefill", "decode_kv8", "block"} <= families
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        record = json.load(f)
    assert families <= set(record["per_launch_dram_bytes"]), families - set(record["per_launch_dram_bytes"])
    assert all(v > 0 for v in record["per_launch_dram_bytes"].values())
