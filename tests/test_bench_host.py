"""bench.py's host-side arithmetic on CPU: the work model behind the roofline line, the traffic
lookup keyed to the kernel sources, the clock-record parsing that decides whether a run is
rejected, and the peaks it divides by. No GPU."""
import json
import os
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from atomistic_neighbor_list_b200 import synth  # noqa: E402


def test_work_model_counts_the_filter_products():
    wl = synth.WORKLOADS["cfg2"]
    E, N = 465_074, 10_000
    bound, fwd, unit = bench.kernel_model("cfconv_fwd_tc", wl, E, N)
    assert (bound, unit) == ("tensor", "TFLOP/s")
    # two layers per edge, R x F then F x F, two FLOP per multiply-add: 45,568 per edge
    assert fwd == 45_568 * E
    bound, bwd, _ = bench.kernel_model("cfconv_bwd_tc", wl, E, N)
    assert bound == "tensor" and bwd == 2 * fwd  # t = e' A1 and v = Q A2 beside z1 and u
    assert bench.kernel_model("cfconv_bwd_simt", wl, E, N)[0] == "alu"


def test_traffic_is_reported_only_for_the_captured_source(tmp_path, monkeypatch):
    entry = {"src_sha": bench.src_digest("cfconv_bwd_tc"), "dram_bytes_per_unit": 15.5}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"cfconv_bwd_tc": entry}))
    real_digest = bench.src_digest("cfconv_bwd_tc")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "src_digest", lambda k: real_digest)
    assert bench.traffic_for("cfconv_bwd_tc", 1000) == pytest.approx(15_500.0)
    assert bench.traffic_for("cfconv_fwd_tc", 1000) is None  # never captured
    monkeypatch.setattr(bench, "src_digest", lambda k: "another-source")
    assert bench.traffic_for("cfconv_bwd_tc", 1000) is None  # kernel changed since the capture


def test_source_digest_follows_every_listed_file():
    d = bench.src_digest("cfconv_fwd_tc")
    assert len(d) == 16 and d == bench.src_digest("cfconv_fwd_tc")
    assert d != bench.src_digest("cfconv_bwd_tc")


def _clocks_from(tmp_path, lines):
    p = tmp_path / "clocks.csv"
    p.write_text("\n".join(lines) + "\n")
    c = object.__new__(bench.Clocks)
    c.path = str(p)
    c.f = open(os.devnull, "w")
    c.proc = types.SimpleNamespace(terminate=lambda: None, wait=lambda timeout=None: 0,
                                   kill=lambda: None)
    return c.stop()


def test_clock_record_median_under_load_and_reasons(tmp_path):
    idle = "0, 345, 1965, 120.5, 0x0, Not Active, Not Active, Not Active, Not Active"
    busy = "0, {}, 1965, 700.0, 0x4, Not Active, Not Active, Not Active, {}"
    rec = _clocks_from(tmp_path, [idle, busy.format(1965, "Not Active"),
                                  busy.format(1950, "Active"), busy.format(1965, "Not Active"),
                                  "garbage line"])
    assert rec["samples"] == 4 and rec["samples_under_load"] == 3  # idle row and junk left out
    assert rec["sm_mhz"] == 1965.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]


def test_clock_record_flags_thermal_slowdown(tmp_path):
    row = "0, 1500, 1965, 800.0, 0x40, Not Active, Active, Not Active, Not Active"
    rec = _clocks_from(tmp_path, [row, row])
    assert rec["reasons"] == ["hw_thermal_slowdown"] and rec["sm_mhz"] == 1500.0


def test_clock_record_without_samples_is_none(tmp_path):
    assert _clocks_from(tmp_path, []) is None


def test_peaks_come_from_the_measured_file():
    p = bench.load_peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        d = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        assert p["source"] == "measured" and p["hbm_gbs"] == d["hbm_gbs"]
        assert p["bf16_tflops_sustained"] <= p["bf16_tflops"]
    else:
        assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0


def test_work_model_of_the_pair_kernel_counts_one_filter_per_pair():
    wl = synth.WORKLOADS["cfg2"]
    E, N = 465_074, 10_000
    _, fwd, _ = bench.kernel_model("cfconv_fwd_tc", wl, E, N)
    bound, pair, unit = bench.kernel_model("cfconv_pair_tc", wl, E, N)
    assert (bound, unit) == ("tensor", "TFLOP/s") and pair == fwd / 2


PEAKS = {"hbm_gbs": 6554.9, "bf16_tflops": 1647.4, "bf16_tflops_sustained": 1381.5,
         "sm_max_mhz": 1965.0, "source": "measured"}


def test_roofline_takes_the_dominant_kernel_against_the_burst_peak():
    wl = synth.WORKLOADS["cfg2"]
    E, N = 465_074, 10_000
    prof = {"cfconv_bwd_tc": {"total_ms": 3.0, "launches": 12},   # 0.25 ms per launch
            "cfconv_fwd_tc": {"total_ms": 1.2, "launches": 12},
            "dense_tc": {"total_ms": 0.5, "launches": 28}}
    clocks = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    r = bench.roofline_of(prof, wl, E, N, PEAKS, clocks, per_unit_ms=6.0)
    assert r["kernel"] == "cfconv_bwd_tc" and r["avg_launch_ms"] == 0.25
    work = 2 * 45_568 * E
    assert r["work_per_launch"] == work
    assert abs(r["achieved"] - work / 0.25e-3 / 1e12) < 1e-9
    assert r["peak"] == 1647.4 and abs(r["frac"] - r["achieved"] / 1647.4) < 1e-12
    assert r["share_of_step"] == 0.5


def test_power_capped_clocks_select_the_sustained_peak_and_alu_peaks_follow_the_clock():
    capped = {"sm_mhz": 1300.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.peak_for("tensor", PEAKS, capped)[0] == 1381.5
    capped_high = {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.peak_for("tensor", PEAKS, capped_high)[0] == 1647.4
    alu, _ = bench.peak_for("alu", PEAKS, None)
    assert abs(alu - 148 * 128 * 2 * 1965e6 / 1e12) < 1e-9
    assert bench.peak_for("hbm", PEAKS, None)[0] == 6554.9
    assert bench.roofline_of({}, synth.WORKLOADS["cfg2"], 1, 1, PEAKS, None) is None
