"""Host logic of bench.py that needs no GPU: the clock-sample summary that goes
into the JSON line's ``clocks`` object, and the roofline denominators."""

import json
import os

import bench


def _sampler_with(tmp_path, lines):
    s = bench.ClockSampler(0)
    path = tmp_path / "clocks.csv"
    path.write_text("\n".join(lines) + "\n")

    class _F:
        name = str(path)
    s.file = _F()
    return s


def test_clock_summary_median_max_and_reasons(tmp_path):
    # nvidia-smi --format=csv,noheader,nounits rows in the sampler's field order:
    # index, clocks.sm, clocks.max.sm, power.draw, reasons bitmask, hw_slowdown,
    # hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
    rows = [
        "0, 1965, 1965, 410.20, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1860, 1965, 998.70, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1830, 1965, 1001.30, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, [N/A], 1965, [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]",   # skipped: no clock
        "garbage",                                                    # skipped: short row
    ]
    s = _sampler_with(tmp_path, rows)
    out = s.summary()
    assert out == {"sm_mhz": 1860.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                   "samples": 3}
    assert not os.path.exists(s.file.name)          # the temporary file is removed


def test_clock_summary_reports_every_slowdown_reason(tmp_path):
    rows = [
        "0, 1200, 1965, 700.0, 0x48, Active, Not Active, Not Active, Not Active",
        "0, 1100, 1965, 700.0, 0x68, Not Active, Active, Active, Not Active",
    ]
    out = _sampler_with(tmp_path, rows).summary()
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert out["sm_mhz"] == 1150.0


def test_clock_summary_without_samples_is_none(tmp_path):
    assert _sampler_with(tmp_path, ["0, [N/A], [N/A], 0, 0, x, x, x, x"]).summary() is None
    s = bench.ClockSampler(0)
    assert s.summary() is None                      # sampler never started


def test_peaks_come_from_the_measured_file_when_present():
    hbm, bf16, bf16_sus, kind = bench._peaks()
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        assert kind == "measured"
        assert (hbm, bf16) == (d["hbm_gbs"], d["bf16_tflops"])
    else:
        assert kind == "fallback" and (hbm, bf16, bf16_sus) == (6650.0, 1590.0, 1400.0)


def test_codec_issue_roofline_needs_a_matching_capture(monkeypatch):
    """The codec half's issue figure uses the instructions per element of a capture
    of the same gm_codec.cu source, and none otherwise."""
    import hashlib
    path = os.path.join(os.path.dirname(bench.__file__), "bit_muon_optimizer_b200", "csrc", "gm_codec.cu")
    sha = hashlib.sha256(open(path, "rb").read()).hexdigest()
    clocks = {"sm_mhz": 1500.0}
    monkeypatch.setattr(bench, "CODEC_INSTR", [{"configs": [4], "source_sha256": "0" * 64,
                                                "thread_instr_per_element": 100.0}])
    assert bench.codec_issue(4, 10 ** 9, 50.0, clocks) is None
    monkeypatch.setattr(bench, "CODEC_INSTR", [{"configs": [4], "source_sha256": sha,
                                                "thread_instr_per_element": 100.0}])
    r = bench.codec_issue(4, 10 ** 9, 50.0, clocks)
    assert r["achieved_tinstr_s"] == 100.0 * 10 ** 9 / 0.05
    assert r["peak_tinstr_s"] == 148 * 4 * 32 * 1500.0e6
    assert abs(r["frac"] - r["achieved_tinstr_s"] / r["peak_tinstr_s"]) < 1e-12
    assert bench.codec_issue(2, 10 ** 9, 50.0, clocks) is None        # another workload
    assert bench.codec_issue(4, 10 ** 9, 50.0, None) is None          # no clock record


def test_ns_auto_picks_gram_for_non_square_shapes():
    """--ns auto: the Gram form exactly where the Gram NS page's FLOP rule favours it
    (aspect ratio above 1), the standard form on square matrices."""
    assert bench.ns_name("auto", 768, 768) == "standard"
    assert bench.ns_name("auto", 2048, 768) == "gram"
    assert bench.ns_name("auto", 3584, 18944) == "gram"
    assert bench.ns_name("standard", 2048, 768) == "standard"
    assert bench.ns_name("gram", 768, 768) == "gram"


def test_sub_batches_split_only_the_largest_groups():
    """Groups above about 1e9 elements are stepped as several calls of equal size
    (at most one matrix apart); smaller groups as one call."""
    import bench
    assert bench.sub_batches(56, 18944, 3584) == 14      # 3.8e9 elements: 4 calls
    assert bench.sub_batches(28, 3584, 18944) == 14      # 1.9e9: 2 calls
    assert bench.sub_batches(56, 3584, 3584) == 56       # 0.72e9: one call
    assert bench.sub_batches(44, 5632, 2048) == 44
    assert bench.sub_batches(1, 65536, 65536) == 1       # one matrix above the limit: one call
    for B, m, n in ((56, 18944, 3584), (57, 18944, 3584), (3, 40000, 40000)):
        c = bench.sub_batches(B, m, n)
        calls = -(-B // c)
        assert 1 <= c <= B and (calls == 1 or c == 1 or c * m * n <= 1.5e9)
