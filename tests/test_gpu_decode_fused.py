"""GPU: the decode fused into the heatmap kernel (gkd_heatmap_decode) against the
two-kernel path (gkd_heatmap then gkd_fuse_decode) on the same inputs.

Both paths fuse the same fp32 accumulator values with the same fp32 arithmetic
and take the first maximal pixel, so idx, xy, score and valid must agree bit
for bit (the two-kernel path is itself checked against the oracle in
test_gpu_parity.py). Covered: the small cases of the heatmap parity tests
(ragged C, K = 128, M = 1, rows valid in one modality only, modalities with
different valid ranges, empty crops, shared kernels), the fp32 path, planted
ties and signed zeros, and all five workloads at full size, every crop.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import bf16_dev, dev, to_dev
from prompt_conditioned_keypoint_b200 import binding as gk
from prompt_conditioned_keypoint_b200 import synthetic as S
from prompt_conditioned_keypoint_b200.head import GkdHead, HeadShape

pytestmark = pytest.mark.gpu


def sync_check():
    torch.cuda.synchronize()
    gk.gkd_check_device_error()


def two_kernel_and_fused(feat, fdt, kern, kdt, mask, B, h, w, C, M, K, shared):
    kbs = 0 if shared else M * K * C
    mbs = 0 if shared else M * K
    H, W = 4 * h, 4 * w
    heat = torch.full((B, M, K, H, W), float("nan"), device=dev())
    gk.gkd_heatmap(feat, fdt, B, h, w, C, 4, kern, kdt, kbs, mask, mbs, M, K, heat)
    ref = [torch.empty((B, K, 2), device=dev()), torch.empty((B, K), device=dev()),
           torch.empty((B, K), dtype=torch.int32, device=dev()), torch.empty((B, K), dtype=torch.uint8, device=dev())]
    gk.gkd_fuse_decode(heat, mask, mbs, B, M, K, H, W, None, *ref)
    got = [torch.full((B, K, 2), 7.0, device=dev()), torch.full((B, K), 7.0, device=dev()),
           torch.full((B, K), 7, dtype=torch.int32, device=dev()),
           torch.full((B, K), 7, dtype=torch.uint8, device=dev())]
    scratch = torch.full((B, K), -1, dtype=torch.int64, device=dev())     # dirty: the call must clear it
    gk.gkd_heatmap_decode(feat, fdt, B, h, w, C, 4, kern, kdt, kbs, mask, mbs, M, K, scratch, *got)
    sync_check()
    return [t.cpu().numpy() for t in ref], [t.cpu().numpy() for t in got]


def assert_same_decode(ref, got):
    rxy, rs, ri, rv = ref
    gxy, gs, gi, gv = got
    np.testing.assert_array_equal(gv, rv)
    np.testing.assert_array_equal(gi, ri)
    np.testing.assert_array_equal(gs.view(np.uint32), rs.view(np.uint32))
    np.testing.assert_array_equal(gxy.view(np.uint32), rxy.view(np.uint32))


CASES = [
    dict(seed=21, B=2, h=24, w=24, C=256, K=80, M=2, feat_dtype="f32", valid="prefix"),
    dict(seed=22, B=3, h=5, w=7, C=200, K=13, M=2, feat_dtype="f32", valid="random"),
    dict(seed=23, B=2, h=24, w=24, C=136, K=17, M=2, feat_dtype="bf16", valid="all", shared=True),
    dict(seed=24, B=1, h=1, w=1, C=8, K=1, M=1, feat_dtype="f32", valid="all"),
    dict(seed=26, B=2, h=3, w=9, C=64, K=128, M=1, feat_dtype="bf16", valid="random"),
    dict(seed=27, B=40, h=8, w=8, C=64, K=20, M=2, feat_dtype="f32", valid="random"),
    dict(seed=28, B=1, h=48, w=48, C=72, K=5, M=2, feat_dtype="f32", valid="prefix"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"s{c['seed']}")
def test_fused_decode_equals_two_kernel_path_bf16(case):
    c = dict(case)
    wl = S.make_case(c.pop("seed"), c.pop("B"), c.pop("h"), c.pop("w"), c.pop("C"), c.pop("K"), c.pop("M"),
                     kern_dtype="bf16", **c)
    if wl.B == 40:
        wl.mask[5] = 0
        wl.mask[6] = 0
        wl.mask[7, 0] = 0                       # text only
        wl.mask[8, 1] = 0                       # visual only
        wl.mask[9, 0, :] = 0
        wl.mask[9, 0, 15:] = 1                  # visual rows 15.. and text rows anywhere: different ranges
    kern = S.random_bf16_rows(case["seed"], (wl.Bk, wl.M, wl.K, wl.C), 1.0 / np.sqrt(wl.C))
    feat = bf16_dev(wl.feat) if wl.feat_dtype == "bf16" else to_dev(wl.feat)
    fdt = gk.GKD_BF16 if wl.feat_dtype == "bf16" else gk.GKD_F32
    ref, got = two_kernel_and_fused(feat, fdt, bf16_dev(kern), gk.GKD_BF16, to_dev(wl.mask), wl.B, wl.h, wl.w,
                                    wl.C, wl.M, wl.K, wl.Bk == 1)
    assert_same_decode(ref, got)


@pytest.mark.parametrize("seed,B,h,w,C,K,M", [(31, 1, 24, 24, 1024, 80, 1), (32, 2, 5, 7, 200, 13, 2),
                                               (33, 3, 6, 9, 96, 40, 2)])
def test_fused_decode_equals_two_kernel_path_f32(seed, B, h, w, C, K, M):
    wl = S.make_case(seed, B, h, w, C, K, M, kern_dtype="f32", valid="random")
    rng = np.random.default_rng(seed)
    kern = (rng.standard_normal((wl.Bk, wl.M, wl.K, wl.C)) / np.sqrt(wl.C)).astype(np.float32)
    ref, got = two_kernel_and_fused(to_dev(wl.feat), gk.GKD_F32, to_dev(kern), gk.GKD_F32, to_dev(wl.mask), B, h, w,
                                    C, M, K, False)
    assert_same_decode(ref, got)


def test_fused_decode_ties_and_signed_zeros():
    """Exact ties and zero peaks: a constant feature map against a one-hot kernel
    gives a constant heatmap (the first pixel wins); a zero kernel row gives
    +0 everywhere, and a row whose two modalities are negatives of each other
    fuses to zeros of both signs (the first pixel's sign is the score's)."""
    B, h, w, C, K, M = 2, 6, 5, 64, 4, 2
    feat = np.zeros((B, h, w, C), np.float32)
    feat[..., 3] = 1.5
    feat[1, 2, 3, 7] = -2.0
    kern = np.zeros((1, M, K, C), np.float32)
    kern[0, 0, 0, 3] = 1.0                     # constant 1.5: a tie everywhere
    kern[0, 1, 0, 3] = 0.5
    kern[0, 0, 2, 7] = 1.0                     # channel 7: zero except one negative bump
    kern[0, 1, 2, 7] = -1.0
    kern[0, 0, 3, 5] = 1.0                     # all-zero channel
    mask = np.ones((1, M, K), np.uint8)
    mask[0, 1, 3] = 0
    bits = S.to_bf16_bits(kern)
    ref, got = two_kernel_and_fused(to_dev(feat), gk.GKD_F32, bf16_dev(bits), gk.GKD_BF16, to_dev(mask), B, h, w, C,
                                    M, K, True)
    assert_same_decode(ref, got)
    assert (got[2][:, 0] == 0).all() and (got[2][:, 3] == 0).all()


def test_all_nan_row_decodes_to_the_first_pixel():
    """NaN inputs are outside the contract, but an all-NaN row must not report an
    index outside the heatmap: both decode paths give idx 0 and a NaN score."""
    B, M, K, H, W = 1, 2, 3, 8, 8
    heat = np.random.default_rng(0).standard_normal((B, M, K, H, W)).astype(np.float32)
    heat[0, :, 1] = np.nan
    mask = np.ones((B, M, K), np.uint8)
    outs = [torch.empty((B, K, 2), device=dev()), torch.empty((B, K), device=dev()),
            torch.empty((B, K), dtype=torch.int32, device=dev()), torch.empty((B, K), dtype=torch.uint8, device=dev())]
    gk.gkd_fuse_decode(to_dev(heat), to_dev(mask), M * K, B, M, K, H, W, None, *outs)
    sync_check()
    xy, score, idx, valid = [t.cpu().numpy() for t in outs]
    assert idx[0, 1] == 0 and valid[0, 1] == 1 and np.isnan(score[0, 1])
    assert xy[0, 1, 0] == np.float32(1 - W) / np.float32(W)
    assert 0 <= idx[0, 0] < H * W and 0 <= idx[0, 2] < H * W


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_workload_fused_decode_every_crop(cfg):
    """Full-size workloads, the launch configuration the benchmark times: every
    crop's decode from the fused path equals the two-kernel path's."""
    torch.cuda.empty_cache()
    wl = S.make_config(cfg)
    shape = HeadShape.of(wl)
    two = GkdHead(shape, dev())
    host = two.host_inputs(wl, pin=False)
    two.upload(host)
    two.forward()
    sync_check()
    ref = [t.cpu().numpy() for t in (two.xy, two.score, two.idx, two.valid)]
    del two
    torch.cuda.empty_cache()
    one = GkdHead(shape, dev(), fused_decode=True)
    one.upload(host)
    one.forward()
    sync_check()
    got = [t.cpu().numpy() for t in (one.xy, one.score, one.idx, one.valid)]
    assert_same_decode(ref, got)
    assert ref[3].sum() > 0
