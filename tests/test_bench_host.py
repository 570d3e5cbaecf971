"""Host logic of bench.py without a GPU: the clock record taken during the timed
region (parsing of fake nvidia-smi output, the verdict on throttling), the
roofline arithmetic, and the peak table's fallback."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
bench = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(bench)


def _row(sm, mx=1965, reasons=("Not Active",) * 4, active="0x0000000000000000"):
    return ", ".join(["0", str(sm), str(mx), "650.00", active, *reasons])


def test_clean_run():
    text = "\n".join([_row(1965)] * 5 + [_row(345)])  # one idle sample before the load
    info = bench.ClockSampler.summarize(text)
    assert info["sm_mhz"] == 1965 and info["sm_max_mhz"] == 1965
    assert info["reasons"] == [] and info["samples"] == 6 and info["verdict"] == "ok"


def test_power_cap_is_kept_and_noted():
    cap = ("Not Active", "Not Active", "Not Active", "Active")
    info = bench.ClockSampler.summarize("\n".join([_row(1320, reasons=cap)] * 4))
    assert info["reasons"] == ["sw_power_cap"] and info["verdict"] == "ok"


def test_thermal_or_hardware_slowdown_is_rejected():
    hw = ("Active", "Not Active", "Not Active", "Not Active")
    th = ("Not Active", "Not Active", "Active", "Active")
    info = bench.ClockSampler.summarize("\n".join([_row(1965), _row(1500, reasons=hw), _row(1400, reasons=th)]))
    assert info["reasons"] == ["hw_slowdown", "sw_power_cap", "sw_thermal_slowdown"]
    assert info["verdict"].startswith("rejected") and "sw_power_cap" not in info["verdict"]


def test_locked_clock_without_reason_is_rejected():
    info = bench.ClockSampler.summarize("\n".join([_row(1200)] * 5))
    assert info["verdict"] == "rejected: SM clock well below max with no reason"


def test_no_samples():
    assert bench.ClockSampler.summarize("") is None
    assert bench.ClockSampler.summarize("garbage line\n") is None


def test_roofline_arithmetic_of_the_bench_workload():
    """Algorithmic bytes and flops of linear + LN B16 H32 T8192: 644 B per head-token
    (Q, K, V bf16 384 B, eta 4 B, Z fp32 256 B) plus W0 in and W_out out (32 KB) per
    unit; 6 d^2 + 4 b d flops per head-token."""
    cfg = bench.I.CONFIGS["linear_ln_B16H32T8192"]
    assert bench.bytes_per_launch(cfg) == 512 * (8192 * 644 + 32768) == 2717908992
    assert bench.flops_per_head_token(cfg) * cfg.head_tokens == 120259084288.0
    mlp = bench.I.CONFIGS["mlp_B8H32T8192"]
    assert bench.flops_per_head_token(mlp) == 14 * 64 * 256 + 4 * 16 * (64 + 256)
    f32 = bench.I.CONFIGS["linear_f32_B1H1T256"]
    assert bench.bytes_per_launch(f32) == 256 * (3 * 256 + 4 + 256) + 32768


def test_peaks_fall_back_when_the_measured_file_is_absent(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, kind = bench.load_peaks()
    assert kind == "fallback" and peaks == bench.FALLBACK_PEAKS
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        '{"hbm_gbs": 6508.8, "bf16_tflops": 1624.0, "bf16_tflops_sustained": 1400.0}')
    peaks, kind = bench.load_peaks()
    assert kind == "measured" and peaks["hbm_gbs"] == 6508.8
