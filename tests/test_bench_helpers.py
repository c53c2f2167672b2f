"""Host-side helpers of bench.py: which peak the roofline divides by, and when
a stored DRAM-traffic figure still belongs to the kernel being timed."""
import importlib.util
import json
import os
import shutil

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(monkeypatch, root):
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    monkeypatch.setattr(b, "ROOT", str(root))
    return b


def _copy_sources(tmp_path):
    dst = tmp_path / "linear_cross_entropy_05_b200" / "csrc"
    shutil.copytree(os.path.join(ROOT, "linear_cross_entropy_05_b200", "csrc"), dst)
    return dst


def test_peaks_come_from_the_measured_file_else_the_stated_fallback(monkeypatch, tmp_path):
    b = _bench(monkeypatch, tmp_path)
    peaks, src = b.measured_peaks()
    assert src == "fallback" and peaks["bf16_tflops_sustained"] == 1400.0 and peaks["hbm_gbs"] == 6650.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"bf16_tflops": 1.0, "bf16_tflops_sustained": 2.0}))
    peaks, src = b.measured_peaks()
    assert src == "measured" and peaks["bf16_tflops_sustained"] == 2.0


def test_source_hash_follows_code_not_comments(monkeypatch, tmp_path):
    csrc = _copy_sources(tmp_path)
    b = _bench(monkeypatch, tmp_path)
    h0 = b.kernel_source_hash("bwd")
    f = csrc / "bwd.cu"
    src = f.read_text()
    f.write_text("// a new comment line\n" + src.replace("namespace cce {", "namespace cce {  /* inline note */", 1))
    assert b.kernel_source_hash("bwd") == h0
    assert b.kernel_source_hash("fwd") != h0          # another kernel's files
    f.write_text(src.replace("constexpr uint32_t TM_S = 0;", "constexpr uint32_t TM_S = 1;", 1))
    assert b.kernel_source_hash("bwd") != h0          # a code change invalidates stored counters


def test_stored_traffic_is_reported_only_for_the_same_kernel_code(monkeypatch, tmp_path):
    _copy_sources(tmp_path)
    b = _bench(monkeypatch, tmp_path)
    (tmp_path / "profiles").mkdir()
    store = {"bwd_kernel": {"w": {"dram_bytes_per_launch": 123.0, "source_hash": b.kernel_source_hash("bwd")}},
             "fwd_lse_kernel": {"w": {"dram_bytes_per_launch": 7.0, "source_hash": "0000000000000000"}}}
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(store))
    assert b.ncu_traffic("bwd_kernel", "w") == 123.0
    assert b.ncu_traffic("fwd_lse_kernel", "w") is None   # captured on other code
    assert b.ncu_traffic("bwd_kernel", "other-workload") is None


def test_launch_count_matches_the_kernels_a_step_runs(monkeypatch, tmp_path):
    # one step = fwd_lse(_pair) + finalize, then with the filter on:
    # cnorm, enorm, blocks, scan, flat_rows, bwd_kernel (the launch list of a
    # profiled step shows these eight); fixed point adds the dloss maximum
    # and the two conversion passes, and with the filter on the clearing of
    # the visited dC accumulator rows
    b = _bench(monkeypatch, tmp_path)
    assert b.launches_per_step(2.0 ** -12, False) == 8
    assert b.launches_per_step(0.0, False) == 3
    assert b.launches_per_step(0.0, True) == 8
    assert b.launches_per_step(2.0 ** -12, True) == 12
    # with the forward's row maxima the filter needs no norm pass (the
    # fixed-point scale still does); the stripe path is one kernel
    assert b.launches_per_step(2.0 ** -12, False, row_max=True) == 6
    assert b.launches_per_step(2.0 ** -12, True, row_max=True) == 12
    assert b.launches_per_step(2.0 ** -12, False, stripes=True) == 3


def test_clock_sampler_reduces_nvml_samples(monkeypatch, tmp_path):
    # a fake NVML: the clock falls under the power cap, one sample shows a
    # thermal slowdown; the summary gives the median, the minimum and every
    # reason seen
    import sys
    import types
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1, nvmlClocksEventReasonHwSlowdown=8, nvmlClocksEventReasonHwThermalSlowdown=64,
        nvmlClocksEventReasonHwPowerBrakeSlowdown=128, nvmlClocksEventReasonSwThermalSlowdown=32,
        nvmlClocksEventReasonSwPowerCap=4)
    seq = [(1965, 0), (1965, 4), (1300, 4), (1250, 4), (1250, 4 | 32)]
    state = {"i": 0}

    def clock(h, which):
        return seq[min(state["i"], len(seq) - 1)][0]

    def reasons(h):
        r = seq[min(state["i"], len(seq) - 1)][1]
        state["i"] += 1
        return r

    fake.nvmlInit = lambda: None
    fake.nvmlDeviceGetHandleByIndex = lambda i: "gpu"
    fake.nvmlDeviceGetHandleByPciBusId = lambda bus: "gpu"
    fake.nvmlDeviceGetClockInfo = clock
    fake.nvmlDeviceGetPowerUsage = lambda h: 900000
    fake.nvmlDeviceGetCurrentClocksEventReasons = reasons
    fake.nvmlDeviceGetMaxClockInfo = lambda h, which: 1965
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    b = _bench(monkeypatch, tmp_path)
    cs = b.ClockSampler(0)
    cs.PERIOD_S = 0.0005
    cs.start()
    import time
    while state["i"] < len(seq):
        time.sleep(0.001)
    out = cs.stop()
    # the last reading repeats after the sequence ends; compare on what was seen
    assert out["sm_max_mhz"] == 1965 and out["sm_mhz_min"] == 1250
    assert out["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]
    assert out["sm_mhz"] <= 1300 and out["power_w_max"] == 900.0 and out["source"].startswith("nvml")
