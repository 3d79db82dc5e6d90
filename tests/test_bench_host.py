"""Host logic of bench.py that runs without a GPU: the clock-sample summary and
the rule that a committed ncu traffic figure is used only for the kernel
source it was captured on."""
import hashlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_clock_summary_median_max_and_reasons():
    c = bench.ClockSampler(None)
    c.lines = [
        "1965, 1965, 610.2, Not Active, Not Active, Not Active, Not Active",
        "1950, 1965, 990.0, Not Active, Not Active, Not Active, Active",
        "[N/A], 1965, 0, Not Active, Not Active, Not Active, Not Active",      # unreadable sample: skipped
        "1935, 1965, 1001.5, Not Active, Not Active, Not Active, Active",
        "garbage",
    ]
    s = c.summary()
    assert s == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_summary_flags_every_slowdown_kind():
    c = bench.ClockSampler(None)
    c.lines = ["1200, 1965, 700, Active, Active, Active, Not Active"]
    assert c.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    c.lines = []
    assert c.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_profiled_traffic_only_for_the_captured_source(tmp_path, monkeypatch):
    csrc = tmp_path / "phase_disaggregated_quantized_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = csrc / "k.cuh"
    src.write_bytes(b"kernel v1\n")
    h = hashlib.sha256(b"kernel v1\n").hexdigest()[:16]
    (tmp_path / "profiles" / "k.md").write_text(
        f"# k\n\ntraffic_source_hash: {h}\ntraffic_bytes_per_launch: 123456\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("k.md", "k.cuh") == 123456.0
    src.write_bytes(b"kernel v2\n")                              # the kernel changed since the capture
    assert bench.profiled_traffic("k.md", "k.cuh") is None
    assert bench.profiled_traffic("absent.md", "k.cuh") is None


def test_committed_profiles_name_a_traffic_figure_for_both_hot_kernels():
    for summary, source in (("nvfp4_gemm_qwen3_8b_prefill.md", "nvfp4_gemm.cuh"),
                            ("w4a16_decode_qwen3_8b.md", "w4a16_gemm.cuh")):
        text = open(os.path.join(ROOT, "profiles", summary)).read()
        assert "traffic_source_hash:" in text and "traffic_bytes_per_launch:" in text
        assert os.path.exists(os.path.join(ROOT, "phase_disaggregated_quantized_b200", "csrc", source))


def test_fp4_peak_is_burst_unless_the_power_cap_was_seen():
    burst, sust = bench.fp4_peaks({"bf16_tflops": 1627.0, "bf16_tflops_sustained": 1401.6})
    assert burst == 1627.0 * 4 and sust == 1401.6 * 4
    assert bench.pick_fp4_peak(burst, sust, [])[0] == burst
    assert bench.pick_fp4_peak(burst, sust, ["hw_slowdown"])[0] == burst
    assert bench.pick_fp4_peak(burst, sust, ["sw_power_cap"])[0] == sust


def test_timed_steps_split_into_repeats():
    assert bench.split_steps(400, 5) == [80] * 5
    assert bench.split_steps(12, 5) == [3, 3, 2, 2, 2]
    assert sum(bench.split_steps(7, 5)) == 7
    assert bench.split_steps(3, 5) == [1, 1, 1]
    m, sd = bench.mean_sd([1.0, 2.0, 3.0])
    assert m == 2.0 and abs(sd - 1.0) < 1e-12
