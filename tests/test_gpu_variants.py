"""GPU parity of the variants beside the graded path, against their own CPU
oracles (oracle/variants.py), on the same seeded inputs.

Fusion by linearity: gkd_norm_fuse_kernels (the mean of a prompt row's
normalised modality rows, rounded once) then gkd_heatmap / gkd_fuse_decode with
one modality. Its heatmaps match variants.head_fused_kernels within the same
per-row bound as the graded contraction, and its decode is bit-exact wherever
the oracle's top-2 margin clears that bound.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import (BF16_TOL, F32_TOL, assert_rows_close, bf16_dev, check_decode_against_margin, dev, to_dev)
from oracle import gkd_oracle as O
from oracle import variants as V
from prompt_conditioned_keypoint_b200 import binding as gk
from prompt_conditioned_keypoint_b200 import synthetic as S
from prompt_conditioned_keypoint_b200.head import GkdHead, HeadShape

pytestmark = pytest.mark.gpu


def sync_check():
    torch.cuda.synchronize()
    gk.gkd_check_device_error()


@pytest.mark.parametrize("out_dt", ["f32", "bf16"])
@pytest.mark.parametrize("M", [1, 2])
def test_norm_fuse_parity(out_dt, M):
    rng = np.random.default_rng(9 + M)
    Bk, K, C = 3, 80, 1280
    rows = rng.standard_normal((Bk, M, K, C)).astype(np.float32)
    rows[0, 0, 4] = 0.0                       # zero row, valid
    mask = (rng.random((Bk, M, K)) < 0.6).astype(np.uint8)
    mask[0, 0, 4] = 1
    mask[1, :, 7] = 0                         # no modality
    out = torch.full((Bk, K, C), 7, dtype=torch.float32 if out_dt == "f32" else torch.int16, device=dev())
    omask = torch.full((Bk, K), 9, dtype=torch.uint8, device=dev())
    gk.gkd_norm_fuse_kernels(to_dev(rows), to_dev(mask), Bk, M, K, C, 1e-12,
                             gk.GKD_F32 if out_dt == "f32" else gk.GKD_BF16, out, omask)
    sync_check()
    khat = O.norm_rows(rows.astype(np.float64), mask)
    ref, rvalid = V.fused_kernel_rows(khat, mask, "f32")
    np.testing.assert_array_equal(omask.cpu().numpy(), rvalid)
    sel = rvalid.reshape(-1) == 1
    if out_dt == "f32":
        got = out.cpu().numpy().astype(np.float64).reshape(-1, C)
        assert_rows_close(got[sel], ref.reshape(-1, C)[sel], F32_TOL, "norm_fuse f32")
        assert np.all(got[~sel] == 0)
    else:
        got = O.bf16_decode(out.cpu().numpy().view(np.uint16)).reshape(-1, C)
        want, _ = V.fused_kernel_rows(khat, mask, "bf16")
        want = want.reshape(-1, C)
        diff = got != want
        assert diff.mean() < 1e-3, diff.mean()      # fp32 mean then bf16 vs fp64 mean then bf16: rare 1-ulp flips
        ulp = np.abs(want[diff]) * 2.0 ** -7
        assert np.all(np.abs(got[diff] - want[diff]) <= ulp + 1e-45)
        assert np.all(got[~sel] == 0)


def run_fused_rows(wl, crops):
    """The fusion-by-linearity head on the GPU for a whole workload; returns the
    heatmaps [B][K][H][W] and decode of the selected crops."""
    head = GkdHead(HeadShape.of(wl), dev(), fuse_rows=True)
    head.upload(head.host_inputs(wl, pin=False))
    head.forward()
    sync_check()
    heat = head.heat[crops, 0].cpu().numpy()
    dec = [t.cpu().numpy()[crops] for t in (head.idx, head.valid, head.xy)]
    return heat, dec


def oracle_rows(wl, crops):
    if wl.support is None:
        return wl.rows.astype(np.float64) if wl.Bk == 1 else wl.rows[crops].astype(np.float64)
    proto = O.pool_prototypes(wl.support[crops], wl.kpts[crops], wl.kmask[crops], wl.sigma, wl.stride)
    rows = np.zeros((len(crops), wl.M, wl.K, wl.C))
    rows[:, 0] = proto
    if wl.M == 2:
        rows[:, 1] = wl.rows[crops, 1]
    return rows


@pytest.mark.parametrize("case", [
    dict(seed=61, B=3, h=24, w=24, C=256, K=80, M=2, feat_dtype="f32", valid="random"),
    dict(seed=62, B=2, h=5, w=7, C=200, K=13, M=2, feat_dtype="bf16", valid="prefix", shared=True),
    dict(seed=63, B=2, h=12, w=12, C=128, K=40, M=1, feat_dtype="f32", valid="all"),
], ids=lambda c: f"s{c['seed']}")
def test_fused_rows_head_small(case):
    c = dict(case)
    wl = S.make_case(c.pop("seed"), c.pop("B"), c.pop("h"), c.pop("w"), c.pop("C"), c.pop("K"), c.pop("M"),
                     kern_dtype="bf16", **c)
    crops = list(range(wl.B))
    heat, (idx, valid, _) = run_fused_rows(wl, crops)
    f64 = O.bf16_decode(wl.feat) if wl.feat_dtype == "bf16" else wl.feat.astype(np.float64)
    href, (_, _, _, _, vref) = V.head_fused_kernels(f64, wl.rows.astype(np.float64), wl.mask, operand="bf16")
    rvalid = np.asarray(wl.mask).any(axis=1)
    rvalid = np.broadcast_to(rvalid, (wl.B, wl.K)) if wl.Bk == 1 else rvalid
    sel = rvalid.reshape(-1)
    assert_rows_close(heat.reshape(-1, wl.H * wl.W)[sel], href.reshape(-1, wl.H * wl.W)[sel], BF16_TOL,
                      "fused-rows heatmaps")
    fref = np.nan_to_num(href, nan=0.0)
    checked, _ = check_decode_against_margin(fref, vref, idx, valid, BF16_TOL, fref[:, None],
                                             rvalid[:, None].astype(np.uint8))
    assert checked > 0


@pytest.mark.parametrize("cfg,crops", [(2, [0, 17, 40, 63]), (3, [0, 101, 255]), (4, [0, 511, 1023]),
                                       (5, [0, 31])], ids=["w2", "w3", "w4", "w5"])
def test_fused_rows_workload(cfg, crops):
    torch.cuda.empty_cache()
    wl = S.make_config(cfg)
    heat, (idx, valid, xy) = run_fused_rows(wl, crops)
    rows = oracle_rows(wl, crops)
    mask = wl.mask if wl.Bk == 1 else wl.mask[crops]
    f64 = O.bf16_decode(wl.feat[crops]) if wl.feat_dtype == "bf16" else wl.feat[crops].astype(np.float64)
    href, (_, _, _, _, vref) = V.head_fused_kernels(f64, rows, mask, operand="bf16")
    rvalid = np.asarray(mask).any(axis=1)
    rvalid = np.broadcast_to(rvalid, (len(crops), wl.K)) if wl.Bk == 1 else rvalid
    sel = rvalid.reshape(-1)
    worst = assert_rows_close(heat.reshape(-1, wl.H * wl.W)[sel], href.reshape(-1, wl.H * wl.W)[sel], BF16_TOL,
                              f"fused-rows workload {cfg}")
    fref = np.nan_to_num(href, nan=0.0)
    checked, near = check_decode_against_margin(fref, vref, idx, valid, BF16_TOL, fref[:, None],
                                                rvalid[:, None].astype(np.uint8))
    assert checked > 0
    print(f"fused rows, workload {cfg}: worst row error {worst:.2e}, {checked} exact peaks, {near} near ties")


# ----------------------------------------------------------------------------- steps either side of the head
def _boxes():
    return np.array([[33, 38, 241, 310], [0, 0, 640, 480], [10.5, 20.25, 110.5, 70.25], [-20, -10, 700, 200],
                     [600, 400, 639.5, 479.75], [5, 5, 5, 50]], np.float32)     # the last is degenerate


def test_preprocess_bit_exact_against_the_oracle():
    """gkd_preprocess does the oracle's fp64 arithmetic in the same order and rounds
    once to fp32: its output equals the oracle's rounded to fp32, bit for bit."""
    from oracle import preprocess as PP
    rng = np.random.default_rng(3)
    H, W = 480, 640
    img = rng.integers(0, 256, (H, W, 3), dtype=np.uint8)
    boxes = _boxes()
    B = len(boxes)
    out = torch.full((B, 3, 384, 384), 5.0, device=dev())
    gk.gkd_preprocess(to_dev(img), H, W, to_dev(boxes), B, 384, out)
    sync_check()
    got = out.cpu().numpy()
    for b in range(B - 1):
        want = PP.preprocess(img, boxes[b].astype(np.float64)).astype(np.float32)
        np.testing.assert_array_equal(got[b].view(np.uint32), want.view(np.uint32))
    pad = PP.normalised_pad().astype(np.float32)
    for c in range(3):
        assert np.all(got[-1, c] == pad[c])          # degenerate box: all pad


def test_preprocess_small_canvas_and_tiny_image():
    from oracle import preprocess as PP
    rng = np.random.default_rng(4)
    img = rng.integers(0, 256, (5, 7, 3), dtype=np.uint8)
    boxes = np.array([[1, 2, 7, 5], [2.5, 0.5, 4.0, 5.5], [-2, -1, 9, 4]], np.float32)
    out = torch.empty((3, 3, 12, 12), device=dev())
    gk.gkd_preprocess(to_dev(img), 5, 7, to_dev(boxes), 3, 12, out)
    sync_check()
    got = out.cpu().numpy()
    for b in range(3):
        want = PP.preprocess(img, boxes[b].astype(np.float64), 12).astype(np.float32)
        np.testing.assert_array_equal(got[b].view(np.uint32), want.view(np.uint32))


def test_roi_to_image_bit_exact_against_the_oracle():
    boxes = _boxes()
    B, K = len(boxes), 80
    rng = np.random.default_rng(5)
    xy = rng.uniform(-1, 1, (B, K, 2)).astype(np.float32)
    xy[:, 0] = 0.0
    xy[:, 1] = -1.0
    xy[:, 2] = 1.0
    W = 96
    cols = np.arange(K) % W
    xy[:, 3:, 0] = ((2 * cols[3:] + 1 - W) / W).astype(np.float32)      # grid-cell centres as decoded
    out = torch.empty((B, K, 2), device=dev())
    gk.gkd_roi_to_image(to_dev(xy), to_dev(boxes), B, K, 384, out)
    sync_check()
    got = out.cpu().numpy()
    for b in range(B - 1):
        want = V.roi_to_image(xy[b].astype(np.float64), tuple(float(v) for v in boxes[b])).astype(np.float32)
        np.testing.assert_array_equal(got[b].view(np.uint32), want.view(np.uint32))
    assert np.isnan(got[-1]).all()


# ----------------------------------------------------------------------------- contract then upsample
CF_TOL = 1e-4   # no bf16 rounding of U on this path: only fp32 accumulation and fp32 lerps differ from fp64


def run_contract_first(wl, kern_bits):
    feat = bf16_dev(wl.feat) if wl.feat_dtype == "bf16" else to_dev(wl.feat)
    kd = bf16_dev(kern_bits)
    heat = torch.full((wl.B, wl.M, wl.K, 4 * wl.h, 4 * wl.w), float("nan"), device=dev())
    G = torch.empty((wl.B, wl.M, wl.K, wl.h * wl.w), device=dev())
    kbs = 0 if wl.Bk == 1 else wl.M * wl.K * wl.C
    mbs = 0 if wl.Bk == 1 else wl.M * wl.K
    gk.gkd_heatmap_contract_first(feat, gk.GKD_BF16 if wl.feat_dtype == "bf16" else gk.GKD_F32, wl.B, wl.h, wl.w,
                                  wl.C, 4, kd, kbs, to_dev(wl.mask), mbs, wl.M, wl.K, G, heat)
    sync_check()
    return heat.cpu().numpy()


@pytest.mark.parametrize("case", [
    dict(seed=71, B=3, h=24, w=24, C=256, K=80, M=2, feat_dtype="f32", valid="random"),
    dict(seed=72, B=2, h=5, w=7, C=200, K=13, M=2, feat_dtype="f32", valid="prefix"),
    dict(seed=73, B=2, h=24, w=24, C=136, K=17, M=2, feat_dtype="bf16", valid="all", shared=True),
    dict(seed=74, B=2, h=3, w=9, C=64, K=128, M=1, feat_dtype="bf16", valid="random"),
    dict(seed=75, B=1, h=48, w=48, C=72, K=5, M=2, feat_dtype="f32", valid="prefix"),
    dict(seed=76, B=5, h=1, w=1, C=8, K=3, M=2, feat_dtype="f32", valid="random"),
    dict(seed=77, B=1, h=160, w=160, C=16, K=4, M=1, feat_dtype="f32", valid="all"),   # source map > 96 KB
], ids=lambda c: f"s{c['seed']}")
def test_contract_first_parity(case):
    from gpu_helpers import valid_heat_rows
    c = dict(case)
    wl = S.make_case(c.pop("seed"), c.pop("B"), c.pop("h"), c.pop("w"), c.pop("C"), c.pop("K"), c.pop("M"),
                     kern_dtype="bf16", **c)
    kern = S.random_bf16_rows(case["seed"], (wl.Bk, wl.M, wl.K, wl.C), 1.0 / np.sqrt(wl.C))
    got = run_contract_first(wl, kern)
    f64 = O.bf16_decode(wl.feat) if wl.feat_dtype == "bf16" else wl.feat.astype(np.float64)
    kf = O.bf16_decode(kern)
    ref = np.stack([V.heatmap_crop_contract_first(f64[b], kf[0 if wl.Bk == 1 else b],
                                                  wl.mask[0 if wl.Bk == 1 else b], 4, "bf16")
                    for b in range(wl.B)])
    g, sel = valid_heat_rows(got, wl.mask)
    r, _ = valid_heat_rows(ref, wl.mask)
    if sel:
        assert_rows_close(g, r, CF_TOL, "contract-first heatmaps")
    mask = np.asarray(wl.mask, bool)
    if mask.shape[0] == 1:
        mask = np.broadcast_to(mask, (wl.B,) + mask.shape[1:])
    assert np.isnan(got[~mask]).all()                   # rows with mask 0 untouched


@pytest.mark.parametrize("cfg,crops", [(2, [0, 33, 63]), (3, [5, 200]), (4, [0, 700]), (5, [0, 31])],
                         ids=["w2", "w3", "w4", "w5"])
def test_contract_first_workload(cfg, crops):
    """Full-size workloads in the benchmark's launch shape: the contract-first
    heatmaps of sampled crops against the variant's oracle. The kernel-row
    operand of every crop is the oracle's normalisation rounded to bf16 (the
    graded normalisation kernel is checked against the same oracle elsewhere)."""
    from gpu_helpers import valid_heat_rows
    torch.cuda.empty_cache()
    wl = S.make_config(cfg)
    allc = list(range(wl.Bk))
    kref = O.bf16_round(O.norm_rows(oracle_rows(wl, allc), wl.mask))
    kbits = (kref.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    got = run_contract_first(wl, kbits)[crops]
    mask = wl.mask if wl.Bk == 1 else wl.mask[crops]
    f64 = O.bf16_decode(wl.feat[crops]) if wl.feat_dtype == "bf16" else wl.feat[crops].astype(np.float64)
    ref = np.stack([V.heatmap_crop_contract_first(f64[i], kref[0 if wl.Bk == 1 else crops[i]],
                                                  mask[0 if wl.Bk == 1 else i], 4, "bf16")
                    for i in range(len(crops))])
    g, sel = valid_heat_rows(got, mask)
    r, _ = valid_heat_rows(ref, mask)
    worst = assert_rows_close(g, r, CF_TOL, f"contract-first workload {cfg}")
    print(f"contract-first workload {cfg}: worst row error {worst:.2e}")
