"""bench.py's host-side bookkeeping on the CPU: the clock summary from
nvidia-smi samples (median SM clock under load, the throttle reasons seen) and
the roofline denominators (the measured peaks, else the fallback figures)."""
import importlib.util
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_host_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _summary(bench, rows):
    s = bench.ClockSampler(0)
    s.f.write("".join(r + "\n" for r in rows))
    return s.summary()


def test_clock_summary_median_under_load_and_reasons():
    bench = _bench()
    idle = "0, 345, 1965, 120.5, 0x0, Not Active, Not Active, Not Active, Not Active"
    load = ["0, {}, 1965, 980.0, 0x4, Not Active, Not Active, Not Active, {}".format(mhz, cap)
            for mhz, cap in ((1965, "Not Active"), (1950, "Active"), (1935, "Active"), (1965, "Not Active"))]
    out = _summary(bench, [idle, idle, idle, idle] + load)
    assert out["samples"] == 8
    assert out["sm_mhz"] == 1957.5          # the upper half of the samples: the loaded ones
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]


def test_clock_summary_flags_slowdowns_and_no_samples():
    bench = _bench()
    rows = ["0, 1200, 1965, 700.0, 0x8, Active, Not Active, Not Active, Not Active",
            "0, 1100, 1965, 700.0, 0x40, Not Active, Active, Active, Not Active"]
    out = _summary(bench, rows)
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert _summary(bench, [])["reasons"] == ["unsampled"]


def test_peaks_measured_else_fallback(tmp_path, monkeypatch):
    bench = _bench()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks() == (6650.0, 1400.0, 1965.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 7000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1450.0, "sm_max_mhz": 1965}))
    assert bench.measured_peaks() == (7000.0, 1450.0, 1965.0, "measured")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 7000.0, "bf16_tflops": 1600.0}))
    assert bench.measured_peaks() == (7000.0, 1600.0, 1965.0, "measured")
    (tmp_path / "MEASURED_PEAKS.json").write_text("{not json")
    assert bench.measured_peaks()[3] == "fallback"


def test_kernel_work_covers_every_traffic_entry():
    """Every kernel with a DRAM figure has an algorithmic-work rule unless it
    is the side kernel (no roofline line of its own), and the tensor-bound
    kernels name a dtype whose peak ratio is known."""
    bench = _bench()
    assert set(bench.DRAM_BYTES_PER_FRAME) - set(bench.KERNEL_WORK) <= {"transform_side"}
    for name, (bound, fn, dtype) in bench.KERNEL_WORK.items():
        assert bound in ("hbm", "tensor"), name
        assert (dtype in bench.TENSOR_RATIO) if bound == "tensor" else dtype is None, name
        assert fn(1.0, 1.0, 1.0) > 0, name
