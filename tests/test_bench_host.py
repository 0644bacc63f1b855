"""bench.py host logic (CPU): the dominant kernel's DRAM traffic is taken from
its committed ncu summary only while the kernel source is the one captured."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_ratio_of_the_committed_capture():
    ratio, src = bench.attn_traffic_ratio()
    assert src.startswith("profiles/"), src
    assert 1.0 <= ratio < 1.1  # DRAM bytes per algorithmic byte of the capture


def test_traffic_is_null_once_the_kernel_changes(tmp_path, monkeypatch):
    changed = tmp_path / "attn.cuh"
    changed.write_bytes(open(bench.ATTN_SOURCE, "rb").read() + b"\n// edited\n")
    monkeypatch.setattr(bench, "ATTN_SOURCE", str(changed))
    ratio, why = bench.attn_traffic_ratio()
    assert ratio is None and "changed" in why


def test_traffic_is_null_without_a_profile(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ATTN_PROFILE", str(tmp_path / "missing.md"))
    assert bench.attn_traffic_ratio() == (None, "no profile")
