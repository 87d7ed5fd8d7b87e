"""Host-side pieces of bench.py: the DRAM counters of a committed ncu summary
are reported only for the CUDA sources they were taken from."""
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _recorded_digest(workload):
    for line in open(os.path.join(ROOT, "profiles", "dram_traffic_%s.txt" % workload)):
        if line.startswith("sources_sha256"):
            return line.split("=", 1)[1].strip()
    raise AssertionError("no sources_sha256 line")


def test_traffic_read_only_for_the_captured_sources(monkeypatch):
    digest = _recorded_digest("b1")
    monkeypatch.setattr(bench, "_sources_digest", lambda: digest)
    t = bench._measured_traffic("b1")
    assert set(t) == {"dense_front", "expert_gate_up", "expert_down", "latent_tail"}
    assert all(v > 1e6 for v in t.values())
    monkeypatch.setattr(bench, "_sources_digest", lambda: "0" * 64)
    assert bench._measured_traffic("b1") == {}


def test_no_summary_no_traffic():
    assert bench._measured_traffic("no-such-workload") == {}


def test_digest_covers_the_cuda_sources_and_header():
    d = bench._sources_digest()
    assert len(d) == 64 and d == bench._sources_digest()
