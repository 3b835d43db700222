"""The measurement records that the benchmark line carries, checked on CPU.

`bench.py` reports a kernel's ncu DRAM traffic from `profiles/traffic.json` only while the record
was taken on the current source (a SHA-256 of the kernel's file); these tests run that rule on a
temporary tree, check that the committed records are per-launch figures close to the algorithmic
bytes of the launch they describe, and that `profiles/` holds text summaries only.
"""
import hashlib
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _tree(tmp_path, src_text, recorded_text):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cu").write_text(src_text)
    rec = {"k": {"dram_bytes_per_launch": 123.0, "source": "k.cu",
                 "source_sha256": hashlib.sha256(recorded_text.encode()).hexdigest(), "captured": "test"}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))


def test_traffic_reported_only_for_the_recorded_source(tmp_path, monkeypatch):
    _tree(tmp_path, "kernel v1\n", "kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic("k") == 123.0
    (tmp_path / "k.cu").write_text("kernel v2\n")  # the kernel changed after the capture
    assert bench._traffic("k") is None
    assert bench._traffic("absent") is None


# algorithmic bytes of one decode launch at the bench workload (B = 8, N = 262,144, d = 128):
# K and V read once plus a 4-byte score per older token (N - 128 of them per sequence)
_B, _N, _D, _W = 8, 262144, 128, 128
_ALGO = {"dec_fused": _B * _N * _D * 2 * 2 + _B * (_N - _W) * 4,
         "dec_fused_e4m3": _B * _N * _D * 2 + _B * (_N - _W) * 4}


@pytest.mark.parametrize("kernel", sorted(_ALGO))
def test_committed_traffic_records_are_per_launch_and_near_the_algorithmic_bytes(kernel):
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)[kernel]
    assert os.path.exists(os.path.join(ROOT, rec["source"]))
    assert len(rec["source_sha256"]) == 64
    # a full launch reads the cache once: within 1% of the algorithmic bytes, never a multiple
    assert abs(rec["dram_bytes_per_launch"] / _ALGO[kernel] - 1.0) < 0.01


def test_profiles_hold_text_summaries_only():
    names = os.listdir(os.path.join(ROOT, "profiles"))
    assert names
    for n in names:
        assert os.path.splitext(n)[1] in (".md", ".txt", ".json"), n
        assert os.path.getsize(os.path.join(ROOT, "profiles", n)) < 64 * 1024, n
