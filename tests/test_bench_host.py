"""Host logic of bench.py, on the CPU: the FLOP and pair counts, the source
hash that guards the committed traffic figure, the traffic lookup, the
clock summary and the peak fallback."""
import json

import numpy as np
import pytest

import bench
import synthetic


def test_visible_pairs_by_brute_force():
    N = 37
    rows = np.array([0, 5, 36], dtype=np.int64)
    causal = sum(1 for i in rows for j in range(N) if j <= i)
    assert bench.visible_pairs(rows, N, True) == causal
    assert bench.visible_pairs(rows, N, False) == len(rows) * N


def test_headline_flop_count():
    # 4 d per visible (query, key) pair: 2 d for Q K^T and 2 d for P V.
    w = synthetic.WORKLOADS["prefill32k"]
    assert w.flops() == pytest.approx(4 * 128 * (32768 * 32769 // 2) * 32)
    assert w.flops() == pytest.approx(8.796e12, rel=1e-3)


def test_source_hash_ignores_comments_and_layout():
    a = 'int f(int x) {\n  // a comment\n  return x + 1; /* another */\n}\nconst char* s = "// kept";\n'
    b = 'int f(int x) { return x + 1; }\nconst char* s = "// kept";'
    c = 'int f(int x) { return x + 2; }\nconst char* s = "// kept";'
    assert bench._strip_comments(a) == bench._strip_comments(b)
    assert bench._strip_comments(b) != bench._strip_comments(c)
    assert '"// kept"' in bench._strip_comments(a)
    h = bench.kernel_source_hash()
    assert len(h) == 16 and h == bench.kernel_source_hash()


def test_traffic_only_for_the_matching_source(tmp_path, monkeypatch):
    summary = tmp_path / "traffic.txt"
    summary.write_text(json.dumps({"kernel_source_hash": "0123456789abcdef", "dram_bytes_per_launch": 42.0}))
    monkeypatch.setattr(bench, "PROFILE_SUMMARY", str(summary))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0123456789abcdef")
    assert bench.traffic_per_launch() == 42.0
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "fedcba9876543210")
    assert bench.traffic_per_launch() is None
    monkeypatch.setattr(bench, "PROFILE_SUMMARY", str(tmp_path / "missing.txt"))
    assert bench.traffic_per_launch() is None


def test_committed_traffic_summary_is_well_formed():
    with open(bench.PROFILE_SUMMARY) as fh:
        s = json.load(fh)
    assert len(s["kernel_source_hash"]) == 16
    assert s["dram_bytes_per_launch"] > 0
    assert "--clock-control none" in s["command"]


def test_clock_summary_parses_nvidia_smi_lines():
    cs = bench.ClockSampler(0)
    cs.lines = [
        "0, 1965, 1965, 700.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1830, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 300, 1965, 100.0, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active",  # idle sample
        "garbage",
    ]
    s = cs.summary()
    assert s["sm_mhz"] == pytest.approx((1965 + 1830) / 2)
    assert s["sm_max_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"] and s["samples"] == 3
    empty = bench.ClockSampler(0)
    empty.lines = []
    assert empty.summary()["reasons"] == ["unavailable"]


def test_peak_falls_back_without_the_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "PEAKS_FILE", str(tmp_path / "absent.json"))
    burst, sustained, src = bench.fp8_peak()
    assert src == "fallback" and burst > sustained > 0
    f = tmp_path / "peaks.json"
    f.write_text(json.dumps({"bf16_tflops": 1000.0, "bf16_tflops_sustained": 900.0}))
    monkeypatch.setattr(bench, "PEAKS_FILE", str(f))
    assert bench.fp8_peak() == (1000.0 * bench.FP8_OVER_BF16, 900.0 * bench.FP8_OVER_BF16, "measured")


@pytest.mark.parametrize("argv,message", [
    (["--impl", "reference", "--path", "bwd"], "--impl reference covers"),
    (["--impl", "reference", "--path", "decode"], "--impl reference covers"),
    (["--shard", "heads", "--path", "wide"], "--shard heads covers"),
    (["--warmup", "2"], "--warmup must be >= 3"),
    (["--seq-len", "4096", "--impl", "reference"], "--seq-len covers"),
    (["--seq-len", "4096", "--shard", "heads"], "--seq-len covers"),
    (["--head-dim", "64", "--path", "bwd"], "--head-dim covers"),
])
def test_dispatch_guards_exit_before_any_device_work(argv, message, monkeypatch):
    monkeypatch.setattr("sys.argv", ["bench.py", *argv])
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    with pytest.raises(SystemExit) as exc:
        bench.main()
    assert message in str(exc.value)


def test_peak_clock_for_the_clock_normalised_fraction(tmp_path, monkeypatch):
    f = tmp_path / "peaks.json"
    f.write_text(json.dumps({"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0,
                             "clocks_under_load": {"sm_mhz_median": 1312.0}}))
    monkeypatch.setattr(bench, "PEAKS_FILE", str(f))
    assert bench.peak_clock_mhz() == 1312.0
    f.write_text(json.dumps({"bf16_tflops": 1600.0}))
    assert bench.peak_clock_mhz() is None
    monkeypatch.setattr(bench, "PEAKS_FILE", str(tmp_path / "missing.json"))
    assert bench.peak_clock_mhz() is None
