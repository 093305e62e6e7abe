"""bench.py reports the fused kernel's measured DRAM traffic only while the
committed capture matches the kernel's current sources and workload; the
figure is the capture's bytes for one layer times the layers a launch walks.
Host logic only (no GPU)."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from synth import synth  # noqa: E402


@pytest.fixture
def repo(tmp_path, monkeypatch):
    """A scratch copy of the repository layout: bench.measured_traffic reads
    profiles/ beside bench.py; the digest stays that of the real sources."""
    digest = bench.kernel_source_digest()
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: digest)
    monkeypatch.setattr(bench, "__file__", str(tmp_path / "bench.py"))
    (tmp_path / "profiles").mkdir()

    def write(workload, digest_):
        rec = {"workload": workload, "dram_bytes_per_layer": 1000.0, "source_digest": digest_}
        (tmp_path / "profiles" / "k_decode_layers.traffic.json").write_text(json.dumps(rec))

    return digest, write


def test_digest_covers_the_fused_kernel_sources():
    d = bench.kernel_source_digest()
    assert len(d) == 16 and int(d, 16) >= 0


def test_traffic_scales_by_layers_when_the_capture_matches(repo):
    digest, write = repo
    write("layer4", digest)
    assert bench.measured_traffic(synth.WORKLOADS["layer4"], 24) == 24000.0
    assert bench.measured_traffic(synth.WORKLOADS["layer4"], 1) == 1000.0


def test_traffic_is_null_after_the_sources_change(repo):
    _, write = repo
    write("layer4", "0" * 16)
    assert bench.measured_traffic(synth.WORKLOADS["layer4"], 24) is None


def test_traffic_is_null_for_another_workload(repo):
    digest, write = repo
    write("layer2", digest)
    assert bench.measured_traffic(synth.WORKLOADS["layer4"], 24) is None


def test_traffic_is_null_without_a_capture(repo):
    assert bench.measured_traffic(synth.WORKLOADS["layer4"], 24) is None
