"""Host-side helpers of bench.py that decide what the JSON line reports.

* ``ncu_traffic``: the DRAM bytes of a committed ncu summary are reported only
  while the kernel sources still hash to the value the summary records;
  after any change to them the traffic field must become null.
* ``ClockSampler.summarise``: median SM clock under load (idle samples below
  the floor dropped), the maximum clock, and every throttle reason that was
  active in any sample.
"""
import os

import bench


def _tree(tmp_path, src_text, summary_text):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cuh").write_text(src_text)
    (tmp_path / "profiles" / "k_ncu.md").write_text(summary_text)


def test_traffic_reported_only_for_the_profiled_sources(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    _tree(tmp_path, "kernel v1\n", "")
    h = bench.source_hash(["k.cuh"])
    (tmp_path / "profiles" / "k_ncu.md").write_text(
        f"| metric | value |\ntraffic_bytes_per_launch: 61684224\nsource_sha256: {h[:16]}\n")
    assert bench.ncu_traffic(["k.cuh"], "k_ncu.md") == 61684224.0
    # the kernel changed after the capture: no traffic figure
    (tmp_path / "k.cuh").write_text("kernel v2\n")
    assert bench.ncu_traffic(["k.cuh"], "k_ncu.md") is None


def test_traffic_absent_without_summary_or_fields(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    _tree(tmp_path, "kernel\n", "no figures here\n")
    assert bench.ncu_traffic(["k.cuh"], "k_ncu.md") is None
    assert bench.ncu_traffic(["k.cuh"], "missing.md") is None


def test_committed_gemm_summary_has_both_fields():
    text = open(os.path.join(bench.ROOT, "profiles", "gemm_flux1024_qkv_ncu.md")).read()
    assert "traffic_bytes_per_launch:" in text and "source_sha256:" in text


def test_clock_summary():
    # timestamp, sm, max sm, power, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
    rows = [
        ["t", "210", "1965", "100", "Not Active", "Not Active", "Not Active", "Not Active"],   # idle: dropped
        ["t", "1950", "1965", "900", "Not Active", "Not Active", "Not Active", "Active"],
        ["t", "1890", "1965", "990", "Not Active", "Not Active", "Not Active", "Active"],
        ["t", "1965", "1965", "800", "Not Active", "Not Active", "Not Active", "Not Active"],
        ["t", "[N/A]", "1965", "800", "Not Active", "Not Active", "Not Active", "Not Active"],  # unparsable
    ]
    s = bench.ClockSampler.summarise(rows)
    assert s["sm_mhz"] == 1950.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    rows.append(["t", "1500", "1965", "1000", "Active", "Not Active", "Active", "Not Active"])
    assert bench.ClockSampler.summarise(rows)["reasons"] == ["hw_slowdown", "sw_power_cap", "sw_thermal_slowdown"]
    assert bench.ClockSampler.summarise([])["sm_mhz"] is None
