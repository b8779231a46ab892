"""bench.py's host-side helpers: the code hash behind the committed DRAM
traffic figures, the gate that drops a figure once the kernel changed, and
the clock record's choice of samples."""
import json

import bench


def test_code_hash_ignores_comments_and_whitespace_but_not_code():
    src = 'int a = 1;  // note\n/* block\n comment */ float b = 2.0f;\n'
    assert bench._code_only(src) == bench._code_only(
        'int a = 1; /* other words */\n\n   float b = 2.0f; // more\n')
    assert bench._code_only(src) != bench._code_only(src.replace("2.0f", "3.0f"))
    # comment markers inside string and character literals are code
    lit = 'const char* s = "// not a comment"; char c = \'/\';'
    assert bench._code_only(lit) == lit
    assert bench._code_only('x = "a\\"b"; // c') == 'x = "a\\"b";'


def test_kernel_hash_covers_every_named_source():
    h1 = bench.kernel_source_hash(("attn_fwd_kernel.cuh",))
    h2 = bench.kernel_source_hash(("attn_fwd_kernel.cuh", "ptx_sm100.cuh"))
    assert len(h1) == 16 and h1 != h2


def test_traffic_figure_is_dropped_when_the_code_changed(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic_w.json").write_text(json.dumps(
        {"kernel_source_hash": "abc", "dram_bytes_per_launch": 123}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda sources=None: "abc")
    assert bench.load_traffic("w") == 123
    monkeypatch.setattr(bench, "kernel_source_hash", lambda sources=None: "def")
    assert bench.load_traffic("w") is None
    assert bench.load_traffic("missing") is None


def _sampler(samples, t0, t1):
    c = bench.ClockSampler(0)
    c.samples = list(samples)
    c.t_begin, c.t_end = t0, t1
    c._stop.set()
    return c


def test_clock_record_keeps_samples_inside_the_region():
    s = [(0.00, 1965.0, 0), (0.02, 1900.0, 0x4), (0.03, 1965.0, 0),
         (0.04, 1965.0, 0), (0.10, 1500.0, 0x40)]
    rec = _sampler(s, 0.015, 0.05).stop()
    assert rec["samples"] == 3 and rec["window"] == "inside the timed region"
    assert rec["sm_mhz"] == 1965.0
    # the power cap seen inside counts; the thermal slowdown after does not
    assert rec["reasons"] == ["sw_power_cap"]
    assert abs(rec["region_ms"] - 35.0) < 1e-6


def test_clock_record_of_a_short_region_takes_the_nearest_samples():
    s = [(0.00, 1900.0, 0), (0.01, 1965.0, 0), (0.03, 1955.0, 0x8), (0.05, 1965.0, 0)]
    rec = _sampler(s, 0.015, 0.02).stop()  # no sample inside
    assert rec["samples"] == 2
    assert rec["window"].startswith("the region's own samples plus")
    # the last sample before and the first after: 1965 and 1955 (hw_slowdown)
    assert rec["sm_mhz"] == 1960.0 and rec["reasons"] == ["hw_slowdown"]


def test_exp_roof_counts_one_exp2_per_visible_score():
    # the headline's count: 32 heads x 16384^2 scores, one exp2 each
    flops = 4.0 * 1 * 32 * 16384 ** 2 * 128
    r = bench.exp_roof(flops, 128, 3.5, 148, 1965.0)
    assert r["exp2_per_launch"] == 32 * 16384 ** 2
    assert abs(r["peak"] - 16 * 148 * 1965e6 / 1e9) < 1e-6
    assert abs(r["achieved"] - 32 * 16384 ** 2 / 3.5e-3 / 1e9) < 1e-3
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12
    assert r["mufu_share"] == 1.0
    # no clock sample: the maximum clock; d = 64 puts an eighth on the FMA pipe
    r64 = bench.exp_roof(flops / 2, 64, 1.0, 148, None)
    assert r64["peak"] == r["peak"] and r64["mufu_share"] == 0.875
    assert r64["exp2_per_launch"] == flops / 2 / 256
