"""The bench's clock record: parsing of the nvidia-smi samples taken during the
timed region, and the verdict on throttling.  No GPU (fake nvidia-smi output)."""
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
