"""Host-side checks of bench.py that need no GPU: the DRAM traffic it reports
for the scored GEMM describes the kernel as the repository builds it."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_recorded_traffic_matches_the_kernel_sources():
    """A recorded ncu traffic figure carries the digest of the sources it was
    captured on; committing a kernel change without a new capture (or without
    clearing the figure) fails here."""
    if bench.NCU_TRAFFIC["bytes"] is None:
        assert bench.ncu_traffic()[0] is None
        return
    assert bench.NCU_TRAFFIC["sources_sha256"] == bench.traffic_sources_digest()
    nbytes, note = bench.ncu_traffic()
    assert nbytes == bench.NCU_TRAFFIC["bytes"] and "ncu" in note


def test_traffic_is_dropped_when_the_sources_change(monkeypatch):
    monkeypatch.setitem(bench.NCU_TRAFFIC, "sources_sha256", "0" * 64)
    monkeypatch.setitem(bench.NCU_TRAFFIC, "bytes", 123)
    assert bench.ncu_traffic() == (None, "kernel sources changed since the capture")


def test_recorded_issue_count_matches_the_kernel_sources():
    """Same rule for the candidate quantiser's recorded instruction count."""
    if bench.NCU_ISSUE["warp_instructions"] is None:
        assert bench.cand_quant_issue(0.3, 1800.0, 148)["warp_instructions"] is None
        return
    assert bench.NCU_ISSUE["sources_sha256"] == bench.issue_sources_digest()


def test_issue_roofline_arithmetic(monkeypatch):
    monkeypatch.setitem(bench.NCU_ISSUE, "warp_instructions", 1_000_000)
    monkeypatch.setitem(bench.NCU_ISSUE, "sources_sha256", bench.issue_sources_digest())
    r = bench.cand_quant_issue(0.5, 1000.0, 100)  # 1e6 / 0.5 ms = 2e9/s; peak 100 x 4 x 1e9
    assert r["bound"] == "alu" and r["frac"] == 0.005
    monkeypatch.setitem(bench.NCU_ISSUE, "sources_sha256", "0" * 64)
    assert bench.cand_quant_issue(0.5, 1000.0, 100)["warp_instructions"] is None
