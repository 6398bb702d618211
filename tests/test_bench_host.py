"""Host-side logic of bench.py, on the CPU: the trimmed mean that averages
the event timer's tick away, the clock record summary (median SM clock,
throttle reasons seen) parsed from nvidia-smi's CSV, and the source hash
that keys the stored ncu traffic figures (comments ignored, code not)."""

import bench


def test_trimmed_mean_drops_a_tenth_each_side():
    xs = [float(v) for v in range(1, 11)]          # 1..10: drop 1 and 10
    assert bench._trimmed_mean(xs) == sum(range(2, 10)) / 8
    assert bench._trimmed_mean([3.0]) == 3.0
    assert bench._trimmed_mean([5.0, 1.0]) == 3.0  # fewer than ten: nothing dropped


def test_trimmed_mean_recovers_a_duration_between_ticks():
    # A 14.85 us kernel read by a timer with 1.024 us ticks: 40 samples of 14 or
    # 15 ticks, in the proportion a uniform phase gives, plus two outliers.
    tick, true_us = 1.024, 14.85
    k = int(true_us // tick)
    frac = true_us / tick - k
    hi = round(40 * frac)
    xs = [k * tick] * (40 - hi) + [(k + 1) * tick] * hi
    xs[0], xs[-1] = 3 * true_us, 0.2 * true_us      # one slow and one bogus read
    got = bench._trimmed_mean(xs)
    assert abs(got - true_us) < 0.1
    median = sorted(xs)[len(xs) // 2]
    assert abs(median - true_us) > 0.3              # the median stays on a tick


def _rows(*rows):
    return "\n".join(", ".join(r) for r in rows) + "\n"


def test_clock_summary_reports_median_clock_and_reasons():
    c = bench.ClockSampler(0)
    na, act = "Not Active", "Active"
    c.out = _rows(
        ("0", "1965", "1965", "700.5", "0x0", na, na, na, na),
        ("0", "1950", "1965", "990.1", "0x4", na, na, na, act),
        ("0", "1965", "1965", "1000.0", "0x4", na, na, na, act),
        ("garbage line",),
    )
    s = c.summary()
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3


def test_clock_summary_flags_thermal_and_missing_samples():
    c = bench.ClockSampler(0)
    na, act = "Not Active", "Active"
    c.out = _rows(("0", "1200", "1965", "800", "0x40", na, act, na, na))
    assert c.summary()["reasons"] == ["hw_thermal_slowdown"]
    c.out = ""
    assert c.summary()["reasons"] == ["unavailable"]


def test_strip_comments_keeps_code_and_literals():
    src = ('int a = 1; // trailing\n'
           'const char* s = "x // not a comment /* nor this */";\n'
           '/* block\n   comment */ char c = \'/\'; char d = \'"\';\n'
           'float e = 2.0f; /**/ int f = a / 2;')
    out = bench._strip_comments(src)
    assert "trailing" not in out and "block" not in out
    assert '"x // not a comment /* nor this */"' in out
    assert "char c = '/';" in out and "char d = '\"';" in out
    assert "int f = a / 2;" in out


def test_hash_ignores_comment_edits_only(tmp_path, monkeypatch):
    csrc = tmp_path / "dequantize_absmax_reduce_b200" / "csrc"
    inc = tmp_path / "include"
    csrc.mkdir(parents=True)
    inc.mkdir()
    for n in bench.TRAFFIC_SOURCES:
        (csrc / n).write_text("int x_%d = 1; // note\n" % len(n))
    (inc / "bq.h").write_text("/* header */ int bq_f(void);\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench._kernel_source_hash()
    (inc / "bq.h").write_text("/* a reworded header comment */ int bq_f(void); // more\n")
    assert bench._kernel_source_hash() == h0
    (inc / "bq.h").write_text("/* header */ int bq_g(void);\n")
    assert bench._kernel_source_hash() != h0
