"""The GPU tests' decode comparison rule, exercised on the CPU with fabricated
device results (no GPU): exact where the oracle's peak is unique, a
near-maximal pixel where it is a near tie, and a failure otherwise."""
import numpy as np
import pytest

from gpu_helpers import BF16_TOL, check_decode_against_margin
from oracle import gkd_oracle as O


def _case(seed, B=3, h=6, w=6, C=16, K=12):
    rng = np.random.default_rng(seed)
    feat = rng.standard_normal((B, h, w, C))
    rows = rng.standard_normal((B, 2, K, C))
    mask = (rng.random((B, 2, K)) < 0.7).astype(np.uint8)
    mask[:, :, 0] = 0
    heat, (fused, idx, xy, score, valid) = O.head(feat, rows, mask, operand="f32")
    return heat, fused, idx, valid, mask


def test_exact_decode_passes_and_counts_every_valid_row():
    heat, fused, idx, valid, mask = _case(1)
    checked, near = check_decode_against_margin(fused, valid, idx, valid, BF16_TOL, heat, mask)
    assert checked + near == int(valid.sum()) and checked > 0


def test_near_tie_accepts_the_runner_up_and_rejects_a_far_pixel():
    heat, fused, idx, valid, mask = _case(2)
    # make row (0, k) a near tie by lifting its runner-up to within the margin
    b, k = 0, int(np.nonzero(valid[0])[0][0])
    f = fused[b, k].reshape(-1)
    p = int(np.argmax(f))
    q = int(np.argsort(f)[-2])
    f[q] = f[p] - 0.1 * BF16_TOL * np.abs(f).max()
    gpu_idx = idx.copy()
    gpu_idx[b, k] = q
    check_decode_against_margin(fused, valid, gpu_idx, valid, BF16_TOL, heat, mask)
    gpu_idx[b, k] = int(np.argmin(f))
    with pytest.raises(AssertionError):
        check_decode_against_margin(fused, valid, gpu_idx, valid, BF16_TOL, heat, mask)


def test_valid_mismatch_and_wrong_unique_peak_fail():
    heat, fused, idx, valid, mask = _case(3)
    bad = valid.copy()
    bad[0, int(np.nonzero(valid[0])[0][0])] = 0
    with pytest.raises(AssertionError):
        check_decode_against_margin(fused, valid, idx, bad, BF16_TOL, heat, mask)
    checked, _ = check_decode_against_margin(fused, valid, idx, valid, BF16_TOL, heat, mask)
    assert checked > 0
    for b in range(fused.shape[0]):
        for k in range(fused.shape[1]):
            f = fused[b, k].reshape(-1)
            if valid[b, k] and O.top2_margin(f) > BF16_TOL * np.abs(f).max():
                gpu_idx = idx.copy()
                gpu_idx[b, k] = (int(idx[b, k]) + 7) % f.size
                with pytest.raises(AssertionError):
                    check_decode_against_margin(fused, valid, gpu_idx, valid, BF16_TOL, heat, mask)
                return
    pytest.fail("no row with a unique peak")


def test_simulated_device_within_tolerance_passes():
    # a stand-in device: every heatmap row off by up to a quarter of the tolerance
    # (the measured bf16 kernel error is at most 5e-4 of the row maximum), then
    # fused and decoded in fp32 like the device path; the rule must accept it
    for trial in range(8):
        heat, fused, idx, valid, mask = _case(100 + trial)
        rng = np.random.default_rng(200 + trial)
        noisy = heat.copy()
        for b in range(heat.shape[0]):
            for m in range(2):
                for k in range(heat.shape[2]):
                    if mask[b, m, k]:
                        S = np.abs(heat[b, m, k]).max()
                        noisy[b, m, k] += rng.uniform(-0.25, 0.25, heat[b, m, k].shape) * BF16_TOL * S
        _, gidx, _, _, gvalid = O.fuse_decode(np.nan_to_num(noisy, nan=0.0).astype(np.float32), mask)
        checked, near = check_decode_against_margin(fused, valid, gidx, gvalid, BF16_TOL, heat, mask)
        assert checked + near == int(valid.sum())


def test_smoke_decode_check_agrees_with_the_test_rule():
    import __graft_entry__ as G
    heat, fused, idx, valid, mask = _case(5)
    exact, near = G.check_decode(fused, heat, mask, idx, BF16_TOL)
    checked, near2 = check_decode_against_margin(fused, valid, idx, valid, BF16_TOL, heat, mask)
    assert (exact, near) == (checked, near2) and exact + near == int(valid.sum())
    b, k = next((b, k) for b in range(valid.shape[0]) for k in range(valid.shape[1]) if valid[b, k])
    bad = idx.copy()
    bad[b, k] = int(np.argmin(fused[b, k]))
    with pytest.raises(AssertionError):
        G.check_decode(fused, heat, mask, bad, BF16_TOL)
