"""Benchmark of the GKDT detection head on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl gkd|reference] [--config 2]

One step = the whole head over one batch of the workload: gkd_norm_kernels ->
gkd_heatmap (fused 4x upsample + 1x1 contraction on tcgen05) ->
gkd_fuse_decode (plus gkd_pool_prototypes on workloads whose visual rows are
pooled). The default workload (2) is a GKDT-L-shaped batch of 64 crops,
C = 1024, 24x24 -> 96x96, dual prompts padded to 80 rows with U{5..80} valid.

For N > 1 (launched by torch.distributed.run) every rank runs its own batch
(weak scaling: crops are independent, no collective on the data path); the
time is the max over ranks. Rank 0 prints one JSON line.

--impl reference times the CPU oracle (the plain fp64 restatement of the head)
on the host cores, on the same workload, each step a bounded sample of it.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "heatmap-head crops/sec (C=1024, 80 prompts, 96×96) and % of roofline, 1 B200"
UNIT = "crops/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
# fp32 FMA peak: 148 SMs x 128 FMA lanes x 2 FLOP x 1.965 GHz (the B200's max SM clock), in TFLOP/s
FFMA_TFLOPS = 148 * 128 * 2 * 1.965 / 1e3


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["gkd", "reference"], default="gkd")
    ap.add_argument("--config", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--e2e-steps", type=int, default=30)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true")
    ap.add_argument("--no-variants", action="store_true")
    ap.add_argument("--per-workload-launches", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-baseline sample")
    return ap.parse_args(argv)


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "MEASURED_PEAKS.json"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_digest() -> str:
    h = hashlib.sha256()
    for name in ("heatmap_tc.cu", "ptx.cuh", "gkd_internal.h"):
        with open(os.path.join(ROOT, "prompt_conditioned_keypoint_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(cfg: int):
    """DRAM bytes per heatmap launch from the committed ncu summary, if it was
    taken on the current kernel source; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    ent = t.get(f"workload{cfg}")
    if not ent or ent.get("kernel_source_digest") != kernel_source_digest():
        return None
    return ent.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Polls NVML (the source nvidia-smi reads) during the timed region."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.index, self.period = index, period_s
        self.samples = []
        self.errors = 0
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:   # no NVML: report it, do not guess
            self.err = str(e)

    def _reasons(self):
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return fn(self.h)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                util = nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                self.samples.append((sm, self._reasons(), util))
            except Exception:   # a failed NVML read: counted and reported, never guessed
                self.errors += 1
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": f"nvml unavailable: {self.err}"}
        busy = [s for s in self.samples if not (s[1] & 0x1)] or self.samples
        bits = 0
        for s in busy:
            bits |= s[1]
        return {"sm_mhz": statistics.median([s[0] for s in busy]) if busy else None, "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in self.REASONS.items() if bits & b and b != 0x1],
                "samples": len(busy), "failed_reads": self.errors}


# ----------------------------------------------------------------------------- CPU oracle legs
def oracle_sample(wl, crop: int, out_rows=None):
    """The oracle head on one crop (optionally a band of output rows)."""
    from oracle import gkd_oracle as O
    f = O.bf16_decode(wl.feat[crop:crop + 1]) if wl.feat_dtype == "bf16" else wl.feat[crop:crop + 1].astype(np.float64)
    kb = 0 if wl.Bk == 1 else crop
    if wl.support is not None:
        proto = O.pool_prototypes(wl.support[crop:crop + 1], wl.kpts[crop:crop + 1], wl.kmask[crop:crop + 1],
                                  wl.sigma, wl.stride)
        rows = np.zeros((1, wl.M, wl.K, wl.C))
        rows[:, 0] = proto
        if wl.M == 2:
            rows[:, 1] = wl.rows[crop:crop + 1, 1]
    else:
        rows = wl.rows[kb:kb + 1].astype(np.float64)
    mask = wl.mask[kb:kb + 1]
    khat = O.norm_rows(rows, mask)
    if wl.kern_dtype == "bf16":
        khat = O.bf16_round(khat)
    heat = O.heatmap_crop(f[0], khat[0], mask[0], wl.up, wl.kern_dtype, out_rows=out_rows)
    return O.fuse_decode(np.nan_to_num(heat, nan=0.0)[None], mask)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(wl, budget_s: float):
    """The oracle as it stands on full crops until the time budget is spent,
    with numpy's BLAS on its default thread pool; plus one crop of workload 1
    with BLAS held to a single thread."""
    n, t0 = 0, time.perf_counter()
    while True:
        oracle_sample(wl, n % wl.B)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= wl.B:
            break
    out = {"value": n / el, "unit": UNIT, "cores": blas_threads(), "host_cores": os.cpu_count(),
           "kind": "oracle",
           "sample": f"{n} full crop(s) of the same workload, fp64 numpy oracle (BLAS matmul for the "
                     f"contraction, {blas_threads()} BLAS threads), {el:.1f} s wall"}
    try:
        from threadpoolctl import threadpool_limits

        from prompt_conditioned_keypoint_b200 import synthetic as S
        w1 = S.make_config(1)
        with threadpool_limits(limits=1, user_api="blas"):
            t1 = time.perf_counter()
            oracle_sample(w1, 0)
            t1 = time.perf_counter() - t1
        out["single_thread_workload1"] = {"value": 1.0 / t1, "unit": UNIT, "cores": 1,
                                          "sample": "the one crop of workload 1, BLAS on one thread"}
    except ImportError:
        out["single_thread_workload1"] = None
    return out


def run_reference(args, cfg_desc):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    from prompt_conditioned_keypoint_b200 import synthetic as S
    wl = S.make_config(args.config)
    H = wl.H
    # size the per-step sample (a band of output rows of one crop) so the whole run stays near two minutes
    t0 = time.perf_counter()
    oracle_sample(wl, 0)
    t_crop = time.perf_counter() - t0
    total_steps = args.steps + args.warmup
    frac = min(1.0, 120.0 / max(total_steps * t_crop, 1e-9))
    nrows = max(1, min(H, int(math.floor(frac * H))))
    sel = list(range(nrows))
    for i in range(args.warmup):
        oracle_sample(wl, i % wl.B, sel)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle_sample(wl, i % wl.B, sel)
    el = time.perf_counter() - t0
    crops = args.steps * nrows / H
    value = crops / el
    sample = f"per step: output rows 0..{nrows - 1} of one crop ({nrows}/{H} of its pixels), fp64 numpy oracle"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": cfg_desc,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------------------- multi-rank timing
def max_over_ranks(seconds: float, pg=None, device="cpu") -> float:
    """The job lasts as long as its slowest rank: max of a per-rank duration."""
    import torch
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    if pg is not None:
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, crops_per_rank: int, steps: int, max_seconds: float) -> float:
    """Whole-job crops/s: every rank processes its own crops_per_rank crops per step."""
    return world * crops_per_rank * steps / max_seconds



# ----------------------------------------------------------------------------- roofline
def heatmap_algorithmic(shape, mask) -> tuple[float, float]:
    """Algorithmic FLOPs and HBM bytes of one gkd_heatmap launch, valid rows only:
    2 R C P FLOPs per crop; bytes = features read once + valid kernel rows
    (bf16, once per distinct prompt set) + valid heatmap rows written (fp32)."""
    m = np.asarray(mask).reshape(np.asarray(mask).shape[0], -1).astype(np.float64)
    rows_per_set = m.sum(axis=1)
    rows_valid = rows_per_set[0] * shape.B if shape.shared else rows_per_set.sum()
    kern_rows = rows_per_set.sum()
    elt = 2 if shape.feat_dtype == "bf16" else 4
    kelt = 2 if shape.kern_dtype == "bf16" else 4
    P = shape.H * shape.W
    flops = 2.0 * rows_valid * shape.C * P
    hbm = shape.B * shape.h * shape.w * shape.C * elt + kern_rows * shape.C * kelt + rows_valid * P * 4
    return flops, hbm


TF32_OVER_BF16 = 1.1 / 2.25        # nominal dense tf32 / bf16 tensor peaks of a B200


def pool_roofline(flops: float, hbm: float, launch_s: float, peaks: dict) -> dict:
    """Gaussian pooling as a tensor-core GEMM (tf32 operands): the bound is the
    slower of its algorithmic FLOPs at the tf32 peak (the measured bf16 peak x
    the nominal tf32/bf16 ratio) and its bytes at the measured HBM peak."""
    peak_tf32 = peaks["bf16_tflops"] * TF32_OVER_BF16
    t_tensor = flops / (peak_tf32 * 1e12)
    t_hbm = hbm / (peaks["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        ach = flops / launch_s / 1e12
        return {"bound": "tensor", "achieved": ach, "peak": peak_tf32, "unit": "TFLOP/s", "frac": ach / peak_tf32,
                "roofline_us": t_tensor * 1e6, "peak_note": "measured bf16 x nominal tf32/bf16"}
    ach = hbm / launch_s / 1e9
    return {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
            "roofline_us": t_hbm * 1e6}


def heatmap_roofline(shape, mask, launch_s: float, peaks: dict) -> dict:
    """Roofline of one gkd_heatmap launch of `launch_s` seconds: bf16 operands
    are bound by the slower of dense bf16 tensor time and HBM time; the fp32
    path by the FFMA rate (148 SMs x 128 lanes x 2 FLOP x 1.965 GHz)."""
    flops, hbm = heatmap_algorithmic(shape, mask)
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = hbm / (peaks["hbm_gbs"] * 1e9)
    achieved = flops / launch_s / 1e12
    if shape.kern_dtype != "bf16":
        peak_alu = FFMA_TFLOPS
        t_alu = flops / (peak_alu * 1e12)
        roof = {"bound": "alu", "achieved": achieved, "peak": peak_alu, "unit": "TFLOP/s",
                "frac": achieved / peak_alu, "roofline_us": max(t_alu, t_hbm) * 1e6}
    elif t_tensor >= t_hbm:
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "roofline_us": t_tensor * 1e6}
    else:
        ach = hbm / launch_s / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "roofline_us": t_hbm * 1e6}
    roof.update({"algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": hbm,
                 "launch_us": launch_s * 1e6, "frac_of_kernel_roofline": roof["roofline_us"] / (launch_s * 1e6)})
    return roof


def per_workload_heatmaps(dev, stream, launches: int, peaks: dict, cfgs=(1, 2, 3, 4, 5)) -> dict:
    """gkd_heatmap alone on each workload at full size: `launches` timed launches
    (CUDA events around each, on the launching stream) after 3 warm-up ones.
    Workload 1 fits in L2, so a 256 MB buffer is written between its launches
    (outside the events); the others move more than L2 per launch."""
    import torch
    from prompt_conditioned_keypoint_b200 import binding as gk
    from prompt_conditioned_keypoint_b200 import synthetic as S
    from prompt_conditioned_keypoint_b200.head import GkdHead, HeadShape
    out = {}
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)
    for cfg in cfgs:
        wl = S.make_config(cfg)
        shape = HeadShape.of(wl)
        head = GkdHead(shape, dev)
        head.upload(head.host_inputs(wl, pin=False), stream)
        with torch.cuda.stream(stream):
            if shape.pooled:
                head.pool(stream)
            head.norm(stream)
            for _ in range(3):
                head.heatmap(stream)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(launches)]
        small = cfg == 1
        for a, b in evs:
            if small:
                with torch.cuda.stream(stream):
                    flush.fill_(1.0)
            a.record(stream)
            head.heatmap(stream)
            b.record(stream)
        stream.synchronize()
        gk.gkd_check_device_error(stream)
        ts = [a.elapsed_time(b) / 1e3 for a, b in evs]
        roof = heatmap_roofline(shape, wl.mask, sum(ts) / len(ts), peaks)
        roof.update({"launch_us_median": 1e6 * statistics.median(ts), "launch_us_min": 1e6 * min(ts),
                     "launches": len(ts), "workload": S.CONFIG_NAMES[cfg],
                     "crops_per_s_heatmap": shape.B / (sum(ts) / len(ts)),
                     "l2": "flushed between launches" if small else "inputs larger than L2"})
        out[f"w{cfg}"] = roof
        del head
        torch.cuda.empty_cache()
    return out


def _time_launches(fn, stream, launches: int, flush=None):
    """Median / mean / min seconds of `fn()` over `launches` timed calls (events on
    `stream`), after 3 warm-up calls; `flush` (if given) runs before each timed call."""
    import torch
    for _ in range(3):
        fn()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(launches)]
    for a, b in evs:
        if flush is not None:
            flush()
        a.record(stream)
        fn()
        b.record(stream)
    stream.synchronize()
    ts = [a.elapsed_time(b) / 1e3 for a, b in evs]
    return statistics.median(ts), sum(ts) / len(ts), min(ts)


def variant_timings(dev, stream, launches: int, peaks: dict, cfg: int = 2) -> dict:
    """The variants beside the graded path, on one workload at full size:
    - fused_decode: whole head with the decode in the heatmap kernel's epilogue
      (norm -> heatmap_decode), crops/s;
    - fuse_rows: fusion by linearity (norm_fuse -> heatmap with M = 1), the
      heatmap launch against its tensor roofline (flops on the fused rows);
    - contract_first: contraction on the source grid + upsample, against HBM
      (features + kernel rows + G written and read + heatmaps written);
    - pool: the pooling kernel on the pooled workloads (1, 5), against the
      slower of its tf32 tensor time and its HBM time;
    - preprocess / roi_to_image: the steps either side of the head, one box per
      crop of the workload (canvases written against HBM; the point map is a
      launch-latency-scale kernel)."""
    import torch
    from prompt_conditioned_keypoint_b200 import binding as gk
    from prompt_conditioned_keypoint_b200 import synthetic as S
    from prompt_conditioned_keypoint_b200.head import GkdHead, HeadShape
    out = {}
    wl = S.make_config(cfg)
    shape = HeadShape.of(wl)
    host = None
    # fused decode: the whole step
    head = GkdHead(shape, dev, fused_decode=True)
    host = head.host_inputs(wl, pin=False)
    head.upload(host, stream)
    with torch.cuda.stream(stream):
        med, mean, mn = _time_launches(lambda: head.forward(stream), stream, launches)
    out["fused_decode"] = {"workload": S.CONFIG_NAMES[cfg], "ms_per_step": 1e3 * mean, "ms_per_step_median": 1e3 * med,
                           "crops_per_s": shape.B / mean,
                           "kernels": "norm, heatmap in decode mode, key finaliser (+ a scratch memset)"}
    del head
    # fusion by linearity: the heatmap launch
    head = GkdHead(shape, dev, fuse_rows=True)
    head.upload(host, stream)
    with torch.cuda.stream(stream):
        if shape.pooled:
            head.pool(stream)
        head.norm(stream)
        med, mean, mn = _time_launches(lambda: head.heatmap(stream), stream, launches)
    fmask = np.asarray(wl.mask).any(axis=1, keepdims=True).astype(np.uint8)
    r = heatmap_roofline(shape, fmask, mean, peaks)
    r.update({"launch_us_median": 1e6 * med, "launch_us_min": 1e6 * mn,
              "note": "flops counted on prompt rows with any modality present (one contraction per row)"})
    out["fuse_rows"] = r
    del head
    # contract then upsample
    head = GkdHead(shape, dev)
    head.upload(host, stream)
    s = shape
    G = torch.empty((s.B, s.M, s.K, s.h * s.w), device=dev)
    kbs = 0 if s.shared else s.M * s.K * s.C
    mbs = 0 if s.shared else s.M * s.K

    def cf():
        gk.gkd_heatmap_contract_first(head.feat, gk.GKD_BF16 if s.feat_dtype == "bf16" else gk.GKD_F32, s.B, s.h,
                                      s.w, s.C, 4, head.khat, kbs, head.mask, mbs, s.M, s.K, G, head.heat, stream)
    with torch.cuda.stream(stream):
        if shape.pooled:
            head.pool(stream)
        head.norm(stream)
        med, mean, mn = _time_launches(cf, stream, launches)
    flops, hbm = heatmap_algorithmic(shape, wl.mask)
    m = np.asarray(wl.mask).reshape(np.asarray(wl.mask).shape[0], -1).astype(np.float64).sum(1)
    rows = m[0] * s.B if s.shared else m.sum()
    hbm_cf = hbm + 2.0 * rows * s.h * s.w * 4          # G written once and read once
    ach = hbm_cf / mean / 1e9
    out["contract_first"] = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": ach / peaks["hbm_gbs"], "launch_us": 1e6 * mean, "launch_us_median": 1e6 * med,
                             "algorithmic_bytes_per_launch": hbm_cf, "algorithmic_flops_per_launch": flops / 16.0,
                             "kernels": "contraction on the source grid (tcgen05) + upsample"}
    del head, G
    torch.cuda.empty_cache()
    # pooling: a tf32 tensor-core GEMM per crop, bound by the slower of its
    # FLOPs at the tf32 peak and its bytes at the HBM peak
    for pc in (1, 5):
        wp = S.make_config(pc)
        hs = HeadShape.of(wp)
        head = GkdHead(hs, dev)
        head.upload(head.host_inputs(wp, pin=False), stream)
        flush = torch.empty(64 << 20, dtype=torch.float32, device=dev) if pc == 1 else None
        with torch.cuda.stream(stream):
            med, mean, mn = _time_launches(lambda: head.pool(stream), stream, launches,
                                           (lambda: flush.fill_(1.0)) if flush is not None else None)
        nk = float(np.asarray(wp.kmask).sum())
        pf = 2.0 * nk * hs.h * hs.w * hs.C
        pb = hs.B * hs.h * hs.w * hs.C * 4 + hs.B * hs.K * hs.C * 4
        out[f"pool_w{pc}"] = dict(pool_roofline(pf, pb, mean, peaks), launch_us=1e6 * mean,
                                  launch_us_median=1e6 * med, algorithmic_flops_per_launch=pf,
                                  algorithmic_bytes_per_launch=pb, hbm_gbs=pb / mean / 1e9)
        del head
    torch.cuda.empty_cache()
    # the steps either side of the head: one 1080p frame, one box per crop of the
    # workload, 384x384 canvases; then the decoded points back to image pixels
    Hi, Wi, canvas = 1080, 1920, 384
    img, boxes = S.random_image_and_boxes(7, Hi, Wi, shape.B)
    img_d = torch.from_numpy(img).to(dev)
    boxes_d = torch.from_numpy(boxes).to(dev)
    canv = torch.empty((shape.B, 3, canvas, canvas), dtype=torch.float32, device=dev)
    with torch.cuda.stream(stream):
        med, mean, mn = _time_launches(lambda: gk.gkd_preprocess(img_d, Hi, Wi, boxes_d, shape.B, canvas, canv, stream),
                                       stream, launches)
    pb = canv.numel() * 4 + img.nbytes          # canvases written once, the frame read once
    ach = pb / mean / 1e9
    out["preprocess"] = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / peaks["hbm_gbs"], "launch_us": 1e6 * mean, "launch_us_median": 1e6 * med,
                         "algorithmic_bytes_per_launch": pb,
                         "workload": f"{shape.B} boxes of a {Wi}x{Hi} RGB frame -> {canvas}x{canvas} fp32 canvases"}
    xy = torch.zeros((shape.B, shape.K, 2), dtype=torch.float32, device=dev)
    pts = torch.empty_like(xy)
    with torch.cuda.stream(stream):
        med, mean, mn = _time_launches(lambda: gk.gkd_roi_to_image(xy, boxes_d, shape.B, shape.K, canvas, pts, stream),
                                       stream, launches)
    out["roi_to_image"] = {"launch_us": 1e6 * mean, "launch_us_median": 1e6 * med,
                           "points_per_launch": shape.B * shape.K, "bound": "launch latency (B K points)"}
    del img_d, boxes_d, canv, xy, pts
    gk.gkd_check_device_error(stream)
    return out


# ----------------------------------------------------------------------------- GPU leg
def main(argv=None):
    args = parse_args(argv)
    rank, local_rank, world = dist_env()
    from prompt_conditioned_keypoint_b200 import synthetic as S
    cfg_desc = {"workload": S.CONFIG_NAMES[args.config], "workload_id": args.config}
    if args.impl == "reference":
        return run_reference(args, cfg_desc)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    import torch
    from prompt_conditioned_keypoint_b200 import binding as gk
    from prompt_conditioned_keypoint_b200.head import GkdHead, HeadPipeline, HeadShape

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pg = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    wl = S.make_config(args.config, shard=rank)
    shape = HeadShape.of(wl)
    head = GkdHead(shape, dev)
    host = head.host_inputs(wl, pin=True)
    stream = torch.cuda.Stream(dev)
    head.upload(host, stream)
    stream.synchronize()

    def barrier():
        if pg:
            pg.barrier()

    # warm-up
    for _ in range(args.warmup):
        head.forward(stream)
    stream.synchronize()
    gk.gkd_check_device_error(stream)

    # timed region: exactly K steps, events on the launching stream
    ev_hm = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(torch.cuda.current_device())
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    t_start.record(stream)
    for i in range(args.steps):
        head.forward(stream, heatmap_events=ev_hm[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks.stop()
    barrier()
    gk.gkd_check_device_error(stream)
    elapsed_s = t_start.elapsed_time(t_end) / 1e3
    hm_list = [a.elapsed_time(b) / 1e3 for a, b in ev_hm]
    hm_s = sum(hm_list) / args.steps

    max_s = max_over_ranks(elapsed_s, pg, dev)
    value = job_throughput(world, shape.B, args.steps, max_s)

    # roofline of the dominant kernel (gkd_heatmap)
    peaks, peak_src = measured_peaks()
    roof = heatmap_roofline(shape, wl.mask, hm_s, peaks)
    flops = roof["algorithmic_flops_per_launch"]
    roof.update({"traffic": committed_traffic(args.config), "kernel": "gkd_heatmap",
                 "peak_source": f"{peak_src} (burst figure)",
                 "launch_us_median": 1e6 * statistics.median(hm_list), "launch_us_min": 1e6 * min(hm_list)})

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * max_s / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": shape.kern_dtype, "data": "synthetic",
            "config": dict(cfg_desc, crops_per_gpu=shape.B, global_batch=world * shape.B, C=shape.C, K=shape.K,
                           M=shape.M, grid=f"{shape.h}x{shape.w}->{shape.H}x{shape.W}",
                           parallelism=f"dp{world} (crops sharded, no data-path collective)",
                           l2="inputs larger than L2 (features + heatmaps per step exceed 126 MB)"),
            "heatmap_gflops": flops / hm_s / 1e9, "roofline": roof,
            "gpu_launches": args.steps * shape.launches_per_step(), "clocks": clocks.summary()}

    # end to end through the public API: pinned host inputs in, decoded keypoints
    # out, every step. Headline: HeadPipeline (two heads; the copy of step i + 1
    # overlaps the head on step i). Also reported: one head, one step after the other.
    if not args.no_e2e:
        def timed_e2e(run_steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier()
            torch.cuda.synchronize(dev)
            e0.record(stream)
            run_steps(e0)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            barrier()
            return max_over_ranks(e0.elapsed_time(e1) / 1e3, pg, dev)

        outh = None
        for _ in range(3):
            outh = head.run_host(host, outh, stream)

        def sequential(_e0):
            for _ in range(args.e2e_steps):
                head.run_host(host, outh, stream)

        t_seq = timed_e2e(sequential)
        pipe = HeadPipeline(shape, dev)
        warm = pipe.run([host] * 3, None, stream)
        outs = [warm[-1]] * args.e2e_steps
        t_pipe = timed_e2e(lambda e0: pipe.run([host] * args.e2e_steps, outs, stream, start_event=e0))
        line["e2e"] = {"value": job_throughput(world, shape.B, args.e2e_steps, t_pipe), "unit": UNIT,
                       "h2d_bytes_per_step": head.host_input_bytes(host), "d2h_bytes_per_step": head.output_bytes(),
                       "steps": args.e2e_steps, "api": "HeadPipeline.run (copies of step i + 1 overlap the head on step i)",
                       "sequential": {"value": job_throughput(world, shape.B, args.e2e_steps, t_seq), "unit": UNIT,
                                      "api": "GkdHead.run_host, one step after the other"}}
        del pipe, warm, outs
    gk.gkd_check_device_error(stream)

    if world == 1 and not args.no_per_workload:
        line["per_workload"] = per_workload_heatmaps(dev, stream, args.per_workload_launches, peaks)
    if world == 1 and not args.no_variants:
        line["variants"] = variant_timings(dev, stream, args.per_workload_launches, peaks)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
