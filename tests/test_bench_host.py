"""bench.py host logic that needs no GPU: the roofline peaks source and the gate on
committed ncu traffic (reported only for the kernel source it was measured on)."""
import json

import bench


def test_traffic_reported_only_for_the_measured_source(tmp_path, monkeypatch):
    path = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.committed_traffic(2) is None                      # no file
    entry = {"dram_bytes_per_launch": 123.0, "kernel_source_digest": bench.kernel_source_digest()}
    path.write_text(json.dumps({"workload2": entry}))
    assert bench.committed_traffic(2) == 123.0
    assert bench.committed_traffic(3) is None                      # other workload: not measured
    entry["kernel_source_digest"] = "0" * 16                        # kernel changed since the capture
    path.write_text(json.dumps({"workload2": entry}))
    assert bench.committed_traffic(2) is None
    path.write_text("{not json")
    assert bench.committed_traffic(2) is None


def test_digest_covers_the_kernel_sources():
    d = bench.kernel_source_digest()
    assert len(d) == 16 and int(d, 16) >= 0


def test_peaks_fallback_when_file_is_missing(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.measured_peaks()
    assert src == "fallback"
    assert peaks["hbm_gbs"] == bench.FALLBACK_HBM_GBS and peaks["bf16_tflops"] == bench.FALLBACK_BF16_TFLOPS
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 1.0, "bf16_tflops": 2.0}))
    peaks, src = bench.measured_peaks()
    assert src == "MEASURED_PEAKS.json" and peaks["bf16_tflops"] == 2.0


def test_args_and_warmup_rule():
    args = bench.parse_args(["--impl", "reference", "--steps", "2", "--warmup", "1"])
    assert args.impl == "reference" and args.steps == 2
    import pytest
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])                              # the GPU leg needs >= 3 warm-up steps


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "1"])
    assert bench.run_reference(args, {"workload": "w", "workload_id": 2}) == 0
    assert capsys.readouterr().out == ""                           # no work, no line on other ranks


def test_clock_sampler_summary_with_a_fake_nvml(monkeypatch):
    """Median SM clock over non-idle samples, union of throttle reasons, and a
    count of failed reads (a stand-in for NVML; no GPU)."""
    import bench

    class FakeNV:
        NVML_CLOCK_SM = 0

        def __init__(self):
            self.calls = 0

        def nvmlDeviceGetClockInfo(self, h, kind):
            self.calls += 1
            if self.calls % 4 == 0:
                raise RuntimeError("transient")
            return 1965 if self.calls % 2 else 1900

        def nvmlDeviceGetCurrentClocksEventReasons(self, h):
            return 0x4 if self.calls % 3 == 0 else 0x0

        def nvmlDeviceGetUtilizationRates(self, h):
            class U:
                gpu = 100
            return U()

    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.samples, cs.errors, cs.period = [], 0, 0.0
    cs.ok, cs.nv, cs.h, cs.max_mhz = True, FakeNV(), None, 1965
    import threading
    cs._stop = threading.Event()
    # run the sampling loop for a fixed number of polls
    polls = {"n": 0}

    def fake_sleep(_):
        polls["n"] += 1
        if polls["n"] >= 12:
            cs._stop.set()

    monkeypatch.setattr(bench.time, "sleep", fake_sleep)
    cs._run()
    s = cs.summary()
    assert s["failed_reads"] == 3 and s["samples"] == 9
    assert s["sm_max_mhz"] == 1965 and s["sm_mhz"] in (1900, 1965)
    assert s["reasons"] == ["sw_power_cap"]


def test_heatmap_roofline_arithmetic():
    """Algorithmic FLOPs and bytes of a heatmap launch count valid rows only
    (shared prompt sets: the rows once per crop for FLOPs and heatmaps, once in
    all for the kernel rows), and the bound is the slower of tensor and HBM time."""
    import numpy as np

    from prompt_conditioned_keypoint_b200.head import HeadShape
    shape = HeadShape(B=2, h=24, w=24, C=1024, K=80, M=2, feat_dtype="f32", kern_dtype="bf16")
    mask = np.zeros((2, 2, 80), np.uint8)
    mask[0, :, :10] = 1          # 20 rows
    mask[1, 0, :5] = 1           # 5 rows
    flops, hbm = bench.heatmap_algorithmic(shape, mask)
    P = 96 * 96
    assert flops == 2.0 * 25 * 1024 * P
    assert hbm == 2 * 576 * 1024 * 4 + 25 * 1024 * 2 + 25 * P * 4
    shared = HeadShape(B=1000, h=24, w=24, C=1024, K=80, M=2, feat_dtype="bf16", kern_dtype="bf16", shared=True)
    m1 = np.zeros((1, 2, 80), np.uint8)
    m1[0, :, :17] = 1
    f2, h2 = bench.heatmap_algorithmic(shared, m1)
    assert f2 == 2.0 * 34 * 1000 * 1024 * P
    assert h2 == 1000 * 576 * 1024 * 2 + 34 * 1024 * 2 + 34 * 1000 * P * 4
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 1.0e6}
    t = flops / 1e15
    r = bench.heatmap_roofline(shape, mask, 2 * t, peaks)
    assert r["bound"] == "tensor" and abs(r["frac"] - 0.5) < 1e-12 and abs(r["roofline_us"] - t * 1e6) < 1e-9
    f32 = HeadShape(B=1, h=24, w=24, C=1024, K=80, M=1, kern_dtype="f32")
    r = bench.heatmap_roofline(f32, mask[:1, :1], 1e-3, peaks)
    assert r["bound"] == "alu"
    slow_hbm = {"bf16_tflops": 1000.0, "hbm_gbs": 1.0}
    r = bench.heatmap_roofline(shape, mask, 1.0, slow_hbm)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and abs(r["achieved"] - hbm / 1e9) < 1e-9


def test_pool_roofline_bound():
    """Pooling is bound by the slower of tf32 tensor time and HBM time."""
    peaks = {"bf16_tflops": 2250.0, "hbm_gbs": 1000.0}
    r = bench.pool_roofline(1.0e9, 1.0e9, 2e-3, peaks)            # HBM: 1 ms; tensor: ~0.9 us
    assert r["bound"] == "hbm" and abs(r["frac"] - 0.5) < 1e-12 and abs(r["roofline_us"] - 1000.0) < 1e-9
    r = bench.pool_roofline(1.1e15, 1.0, 2.0, peaks)              # tensor: 1 s at 1100 TFLOP/s
    assert r["bound"] == "tensor" and abs(r["peak"] - 1100.0) < 1e-6 and abs(r["frac"] - 0.5) < 1e-9
