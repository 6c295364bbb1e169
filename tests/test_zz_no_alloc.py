"""GPU: the decode fused into the heatmap kernel, called through the entry point
that allocates nothing (gkd_heatmap_decode_noalloc), against the entry point
that takes the caller's scratch buffer (gkd_heatmap_decode).

The allocation-free entry point is for callers that are handed only their
inputs and outputs and cannot allocate device memory: its peak keys live in a
statically sized buffer inside the library. Its outputs must equal the other
entry point's bit for bit. Two calls in a row on different inputs check that
each call clears what it uses of the shared buffer (the second call must not
see the first call's keys). This file is named to be collected last; it also
passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import bf16_dev, dev, to_dev
from prompt_conditioned_keypoint_b200 import binding as gk
from prompt_conditioned_keypoint_b200 import synthetic as S

pytestmark = pytest.mark.gpu


def _outputs(B, K):
    return [torch.full((B, K, 2), 7.0, device=dev()), torch.full((B, K), 7.0, device=dev()),
            torch.full((B, K), 7, dtype=torch.int32, device=dev()),
            torch.full((B, K), 7, dtype=torch.uint8, device=dev())]


def _case(seed, B, h, w, C, K, M, feat_dtype, valid, shared=False):
    wl = S.make_case(seed, B, h, w, C, K, M, feat_dtype=feat_dtype, kern_dtype="bf16", valid=valid, shared=shared)
    kern = S.random_bf16_rows(seed, (wl.Bk, wl.M, wl.K, wl.C), 1.0 / np.sqrt(wl.C))
    feat = bf16_dev(wl.feat) if feat_dtype == "bf16" else to_dev(wl.feat)
    fdt = gk.GKD_BF16 if feat_dtype == "bf16" else gk.GKD_F32
    kbs = 0 if shared else M * K * C
    mbs = 0 if shared else M * K
    args = (feat, fdt, B, h, w, C, 4, bf16_dev(kern), gk.GKD_BF16, kbs, to_dev(wl.mask), mbs, M, K)
    return args, B, K


def _both(args, B, K):
    ref = _outputs(B, K)
    scratch = torch.empty((B, K), dtype=torch.int64, device=dev())
    gk.gkd_heatmap_decode(*args, scratch, *ref)
    got = _outputs(B, K)
    gk.gkd_heatmap_decode_noalloc(*args, *got)
    torch.cuda.synchronize()
    gk.gkd_check_device_error()
    return [t.cpu().numpy() for t in ref], [t.cpu().numpy() for t in got]


def _assert_same(ref, got):
    for r, g in zip(ref, got):
        assert r.dtype == g.dtype
        np.testing.assert_array_equal(g.view(np.uint8), r.view(np.uint8))


def test_noalloc_decode_equals_scratch_decode_two_calls_in_a_row():
    first = _case(81, B=12, h=24, w=24, C=256, K=80, M=2, feat_dtype="f32", valid="random")
    second = _case(82, B=5, h=12, w=20, C=136, K=17, M=2, feat_dtype="bf16", valid="all", shared=True)
    for args, B, K in (first, second):
        ref, got = _both(args, B, K)
        _assert_same(ref, got)
        assert ref[3].sum() > 0


def test_noalloc_decode_workload_size_twice():
    """Workload 2's batch shape (64 crops x 80 rows, 5120 keys) twice: the
    second call reuses the buffer the first one filled."""
    wl = S.make_config(2, crops=range(16))
    rows = torch.from_numpy(wl.rows).to(dev())
    mask = to_dev(wl.mask)
    khat = torch.empty((wl.B, wl.M, wl.K, wl.C), dtype=torch.int16, device=dev())
    gk.gkd_norm_kernels(rows, mask, wl.B, wl.M, wl.K, wl.C, 1e-12, gk.GKD_BF16, khat)
    args = (to_dev(wl.feat), gk.GKD_F32, wl.B, wl.h, wl.w, wl.C, 4, khat, gk.GKD_BF16, wl.M * wl.K * wl.C, mask,
            wl.M * wl.K, wl.M, wl.K)
    for _ in range(2):
        ref, got = _both(args, wl.B, wl.K)
        _assert_same(ref, got)
