"""Host-side logic of bench.py that needs no GPU: the peak used as the
roofline denominator, and the rule that DRAM traffic from a committed ncu
capture is reported only while the kernel sources match the capture."""
import json
import os

import bench


def test_measured_peak_prefers_the_driver_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 1234.5}))
    assert bench.measured_peaks() == (1234.5, "measured")


def test_traffic_is_reported_only_for_matching_sources(tmp_path, monkeypatch):
    """A committed DRAM-traffic figure is reported while the files its record
    names are unchanged, and dropped once one of them changes; files outside
    the record's list do not matter."""
    pkg = tmp_path / "hadamard_incoherence_transforms_b200"
    (pkg / "csrc").mkdir(parents=True)
    (pkg / "csrc" / "k.cu").write_text("kernel v1")
    (pkg / "csrc" / "other.cu").write_text("unrelated")
    (pkg / "build.py").write_text("flags")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    srcs = ["csrc/k.cu", "build.py"]
    digest = bench.source_digest(srcs)
    assert len(digest) == 16 and digest == bench.source_digest(srcs)
    rec = {"k": {"dram_bytes_per_launch": 42.0, "sources": srcs, "source_digest": digest}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.read_profile_traffic("k") == 42.0
    assert bench.read_profile_traffic("other") is None
    (pkg / "csrc" / "other.cu").write_text("changed, but not the kernel's")
    assert bench.read_profile_traffic("k") == 42.0
    (pkg / "csrc" / "k.cu").write_text("kernel v2")
    assert bench.read_profile_traffic("k") is None


def test_committed_traffic_record_names_the_headline_kernel():
    path = os.path.join(bench.ROOT, "profiles", "traffic.json")
    with open(path) as f:
        rec = json.load(f)
    assert "k_rows_stream<12,float,float,EPI_QUANT,4>" in rec
    r = rec["k_rows_stream<12,float,float,EPI_QUANT,4>"]
    assert r["dram_bytes_per_launch"] == r["dram_read"] + r["dram_write"]
    # the record names the kernel's translation unit: k_stream.cu and everything it includes
    for f in ("csrc/k_stream.cu", "csrc/rows_stream.cuh", "csrc/rows_ops.cuh", "csrc/rows.cuh", "csrc/device.cuh",
              "csrc/internal.h", "csrc/kernels.h", "build.py"):
        assert f in r["sources"], f


def test_reference_arm_prints_one_contract_line(capsys):
    """The reference arm (the oracle on host cores) runs without a GPU and prints
    the JSON line with the keys the driver reads."""
    assert bench.main(["--impl", "reference", "--steps", "3", "--warmup", "3"]) == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 3 and d["warmup"] == 3 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in d["config"]


def test_reference_arm_is_silent_on_other_ranks(capsys):
    class Args:
        workload, steps, warmup = "weight_rht_int4", 3, 3

    assert bench.run_reference(Args(), 2, 1) == 0
    assert capsys.readouterr().out == ""


def test_clock_sampler_with_a_fake_nvml(monkeypatch):
    """The sampler reads SM clocks and throttle reasons through NVML; a fake
    module stands in for it on a machine without a GPU."""
    import sys
    import time
    import types

    state = {"n": 0}
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByIndex=lambda i: ("h", i),
        nvmlDeviceGetMaxClockInfo=lambda h, kind: 1965,
    )

    def clock(h, kind):
        state["n"] += 1
        return 1965 if state["n"] % 3 else 1800

    fake.nvmlDeviceGetClockInfo = clock
    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x1 | 0x4   # idle (ignored) + power cap
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES", raising=False)
    with bench.ClockSampler(0) as clk:
        time.sleep(0.05)
    out = clk.summary()
    assert out["sm_max_mhz"] == 1965 and out["samples"] >= 5
    assert out["sm_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]


def test_clock_sampler_without_nvml(monkeypatch):
    import sys

    monkeypatch.setitem(sys.modules, "pynvml", None)   # import fails
    with bench.ClockSampler(0) as clk:
        pass
    assert clk.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_clock_sampler_reports_only_the_timed_window(monkeypatch):
    """Samples taken while the sampler starts up (before the timed region)
    are not part of the summary."""
    import sys
    import time
    import types

    state = {"n": 0}

    def clock(h, kind):
        state["n"] += 1
        return 1000 if state["n"] <= 2 else 1965   # the start-up samples read 1000 MHz

    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByIndex=lambda i: ("h", i),
        nvmlDeviceGetMaxClockInfo=lambda h, kind: 1965,
        nvmlDeviceGetClockInfo=clock,
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: 0,
    )
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES", raising=False)
    with bench.ClockSampler(0) as clk:
        time.sleep(0.02)
    out = clk.summary()
    assert out["samples"] >= 3 and out["sm_mhz"] == 1965 and out["reasons"] == []
    assert len(clk.samples) > out["samples"]   # the start-up samples were taken, then left out
