"""bench.py reports an ncu DRAM-traffic figure only while the kernel source
it was captured from is unchanged (host logic; no GPU)."""
import hashlib
import json
import os

import pytest

import bench


def _write(tmp_path, src_bytes, recorded_hash):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cu").write_bytes(src_bytes)
    rec = {"source_files": ["k.cu"], "source_sha256": recorded_hash,
           "kernels": {"tc_qlinear_dx": {"dram_bytes_per_launch": 1234}}}
    (tmp_path / "profiles" / "tc_qlinear_traffic_w.json").write_text(json.dumps(rec))


def test_traffic_reported_when_source_matches(tmp_path, monkeypatch):
    src = b"__global__ void k() {}\n"
    _write(tmp_path, src, hashlib.sha256(src).hexdigest())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("w", "tc_qlinear_dx") == 1234
    assert bench.measured_traffic("w", "tc_qlinear_fwd") is None
    assert bench.measured_traffic("other", "tc_qlinear_dx") is None


def test_traffic_dropped_when_source_changed(tmp_path, monkeypatch):
    _write(tmp_path, b"__global__ void k() { /* edited */ }\n",
           hashlib.sha256(b"__global__ void k() {}\n").hexdigest())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("w", "tc_qlinear_dx") is None
