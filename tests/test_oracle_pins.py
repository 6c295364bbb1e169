"""Pins of the CPU oracle to facts other than itself (CPU only).

Each test ties one oracle function to a closed form, an invariant, a library
routine the step reduces to, a hand-computed golden value, or the pure-Python
brute force on tiny inputs, so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one of them.
"""
import math
import os
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import read_golden
from oracle import brute
from oracle import gkd_oracle as O

RNG = np.random.default_rng(12345)


def f32_from_fraction(q: Fraction) -> np.float32:
    """Correctly rounded fp32 of an exact rational (ties to even), by integer arithmetic."""
    if q == 0:
        return np.float32(0.0)
    sign = -1 if q < 0 else 1
    q = abs(q)
    e = q.numerator.bit_length() - q.denominator.bit_length()
    if Fraction(2) ** e > q:
        e -= 1
    # q in [2^e, 2^(e+1)); fp32 spacing 2^(e-23)
    scaled = q / Fraction(2) ** (e - 23)
    n = scaled.numerator // scaled.denominator
    rem = scaled - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return np.float32(sign * math.ldexp(n, e - 23))


# ---------------------------------------------------------------------------
# bf16 rounding
# ---------------------------------------------------------------------------
def test_bf16_round_matches_torch_on_fp32_inputs():
    x = np.concatenate([
        RNG.standard_normal(20000).astype(np.float32),
        (RNG.standard_normal(2000) * 1e-30).astype(np.float32),
        (RNG.standard_normal(2000) * 1e30).astype(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, 1e-39, -1e-40], np.float32),
    ])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_round(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_bf16_round_ties_even_without_double_rounding():
    one = 1.0
    cases = [
        (one + 2.0 ** -8, one),                        # halfway -> even (1.0)
        (one + 3 * 2.0 ** -8, one + 2.0 ** -6),        # halfway -> even (1 + 2^-6)
        (one + 2.0 ** -8 + 2.0 ** -40, one + 2.0 ** -7),  # above halfway in fp64; via fp32 it would tie down
        (-(one + 2.0 ** -8 + 2.0 ** -40), -(one + 2.0 ** -7)),
        (one + 2.0 ** -8 - 2.0 ** -40, one),
        (3.5e38, np.inf),
    ]
    for x, want in cases:
        assert O.bf16_round(np.array([x]))[0] == want, x


def test_bf16_decode_exact():
    bits = np.array([0x3F80, 0xBF80, 0x0000, 0x8000, 0x4049, 0x0001], np.uint16)
    want = np.array([1.0, -1.0, 0.0, -0.0, 3.140625, 2.0 ** -133])
    np.testing.assert_array_equal(O.bf16_decode(bits), want)


# ---------------------------------------------------------------------------
# a3: bilinear upsample
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("h,w", [(1, 1), (1, 3), (2, 2), (3, 5), (24, 24), (7, 48)])
def test_upsample_matches_torch_interpolate(h, w):
    C = 3
    F = RNG.standard_normal((h, w, C))
    ref = torch.nn.functional.interpolate(
        torch.from_numpy(F.transpose(2, 0, 1)[None].copy()), scale_factor=4, mode="bilinear",
        align_corners=False)[0].numpy().transpose(1, 2, 0)
    got = O.upsample(F, 4)
    assert got.shape == (4 * h, 4 * w, C)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-13)


def test_upsample_constant_map_exact():
    for v in (1.0, 3.25, -0.0078125, float(O.bf16_decode(np.array([0x4049]))[0])):
        F = np.full((24, 24, 2), v)
        U = O.upsample(F, 4)
        assert np.all(U == v)


def test_interp_weights_are_dyadic_and_sum_to_one():
    R = O.interp_matrix(24, 4)
    np.testing.assert_array_equal(R.sum(axis=1), np.ones(96))
    allowed = {0.0, 0.125, 0.375, 0.625, 0.875, 1.0}
    assert set(np.unique(R).tolist()) <= allowed
    # interior pattern d = 4i + r
    i = 10
    assert R[4 * i + 0, i - 1] == 0.375 and R[4 * i + 0, i] == 0.625
    assert R[4 * i + 1, i - 1] == 0.125 and R[4 * i + 1, i] == 0.875
    assert R[4 * i + 2, i] == 0.875 and R[4 * i + 2, i + 1] == 0.125
    assert R[4 * i + 3, i] == 0.625 and R[4 * i + 3, i + 1] == 0.375
    assert R[0, 0] == 1.0 and R[1, 0] == 1.0 and R[94, 23] == 1.0 and R[95, 23] == 1.0


def test_upsample_onehot_golden(golden_dir):
    g = read_golden(os.path.join(golden_dir, "upsample_onehot.txt"))
    h, w, up = int(g["h"][0]), int(g["w"][0]), int(g["up"][0])
    for tag in ("interior", "corner"):
        y0, x0 = map(int, g[f"{tag}_cell"])
        F = np.zeros((h, w, 1))
        F[y0, x0, 0] = 1.0
        kern = np.ones((1, 1, 1))
        heat = O.heatmap_crop(F, kern, np.ones((1, 1), np.uint8), up, "f32")
        if tag == "interior":
            peak = int(g["interior_peak_num"][0]) / int(g["interior_peak_den"][0])
        else:
            peak = float(g["corner_peak"][0])
        assert heat.max() == peak
        rows = list(map(int, g[f"{tag}_peak_rows"]))
        cols = list(map(int, g[f"{tag}_peak_cols"]))
        ys, xs = np.nonzero(heat[0, 0] == peak)
        assert sorted(set(ys.tolist())) == rows and sorted(set(xs.tolist())) == cols
        assert len(ys) == 4
        _, idx, _, _, _ = O.fuse_decode(heat[None].astype(np.float32), np.ones((1, 1, 1), np.uint8))
        assert idx[0, 0] == int(g[f"{tag}_first_index"][0])


def test_upsample_matches_brute_force():
    for h, w in [(1, 1), (2, 3), (4, 4), (3, 1)]:
        C = 3
        F = RNG.standard_normal((h, w, C))
        U = O.upsample(F, 4)
        Fl = F.tolist()
        for Y in range(4 * h):
            for X in range(4 * w):
                for c in range(C):
                    assert abs(U[Y, X, c] - brute.up_value(Fl, h, w, c, Y, X, 4)) < 1e-13


def test_upsample_is_linear():
    F, G = RNG.standard_normal((2, 5, 6, 4))
    a, b = 1.7, -0.3
    np.testing.assert_allclose(O.upsample(a * F + b * G), a * O.upsample(F) + b * O.upsample(G),
                               rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# a4: contraction
# ---------------------------------------------------------------------------
def test_unit_kernel_against_identical_feature_gives_one():
    C = 64
    f = RNG.standard_normal(C)
    F = np.broadcast_to(f, (24, 24, C)).copy()
    k = O.norm_rows(f[None, None, None, :], np.ones((1, 1, 1), np.uint8))[0]
    heat = O.heatmap_crop(F, k, np.ones((1, 1), np.uint8), 4, "f32")
    np.testing.assert_allclose(heat, np.linalg.norm(f), rtol=1e-14)
    funit = f / np.linalg.norm(f)
    F1 = np.broadcast_to(funit, (24, 24, C)).copy()
    heat1 = O.heatmap_crop(F1, k, np.ones((1, 1), np.uint8), 4, "f32")
    np.testing.assert_allclose(heat1, 1.0, rtol=1e-14)


def test_contract_then_upsample_equals_upsample_then_contract():
    h, w, C, K = 6, 5, 16, 3
    F = RNG.standard_normal((h, w, C))
    kern = RNG.standard_normal((1, K, C))
    heat = O.heatmap_crop(F, kern, np.ones((1, K), np.uint8), 4, "f32")
    for k in range(K):
        G = (F @ kern[0, k])[:, :, None]            # contract on the source grid
        Gu = O.upsample(G, 4)[:, :, 0]              # then upsample
        np.testing.assert_allclose(heat[0, k], Gu, rtol=0, atol=1e-12 * np.abs(Gu).max())


def _brute_bf16(x: float) -> float:
    """Independent fp64 -> bf16 rounding (frexp + Python's half-even round)."""
    if x == 0.0 or not math.isfinite(x):
        return x
    m, e = math.frexp(x)
    q = math.ldexp(1.0, max(e - 8, -133))
    return round(x / q) * q


@pytest.mark.parametrize("operand", ["f32", "bf16"])
def test_heatmap_matches_brute_force_tiny(operand):
    rnd = _brute_bf16 if operand == "bf16" else None
    for trial in range(6):
        h, w = int(RNG.integers(1, 5)), int(RNG.integers(1, 5))
        C, K, M = int(RNG.integers(1, 9)), int(RNG.integers(1, 4)), int(RNG.integers(1, 3))
        F = RNG.standard_normal((h, w, C))
        kern = RNG.standard_normal((M, K, C))
        mask = (RNG.random((M, K)) < 0.7).astype(np.uint8)
        heat = O.heatmap_crop(F, kern, mask, 4, operand)
        Fl = F.tolist()
        for m in range(M):
            for k in range(K):
                if not mask[m, k]:
                    assert np.all(np.isnan(heat[m, k]))
                    continue
                for Y in range(4 * h):
                    for X in range(4 * w):
                        ref = brute.heat_value(Fl, h, w, C, kern[m, k].tolist(), Y, X, 4, rnd)
                        assert abs(heat[m, k, Y, X] - ref) <= 1e-12 * max(1.0, abs(ref))


def test_shared_kernels_equal_replicated():
    B, h, w, C, K = 3, 3, 4, 8, 2
    F = RNG.standard_normal((B, h, w, C))
    kern = RNG.standard_normal((1, 2, K, C))
    mask = np.ones((1, 2, K), np.uint8)
    a = O.heatmaps(F, kern, mask, 4, "f32")
    b = O.heatmaps(F, np.repeat(kern, B, 0), np.repeat(mask, B, 0), 4, "f32")
    np.testing.assert_array_equal(a, b)


# ---------------------------------------------------------------------------
# a2: normalisation
# ---------------------------------------------------------------------------
def test_norm_matches_torch_normalize_and_masks():
    rows = RNG.standard_normal((3, 2, 5, 33))
    rows[0, 1, 2] = 0.0
    mask = (RNG.random((3, 2, 5)) < 0.7).astype(np.uint8)
    mask[0, 1, 2] = 1
    got = O.norm_rows(rows, mask)
    ref = torch.nn.functional.normalize(torch.from_numpy(rows), dim=-1, eps=1e-12).numpy()
    np.testing.assert_allclose(got[mask == 1], ref[mask == 1], rtol=1e-15, atol=0)
    assert np.all(got[mask == 0] == 0)
    assert np.all(got[0, 1, 2] == 0)
    n = np.linalg.norm(got, axis=-1)
    valid = (mask == 1) & (np.linalg.norm(rows, axis=-1) > 0)
    np.testing.assert_allclose(n[valid], 1.0, rtol=1e-15)


def test_norm_matches_brute_force():
    rows = RNG.standard_normal((1, 1, 4, 7))
    got = O.norm_rows(rows, np.ones((1, 1, 4), np.uint8))
    for k in range(4):
        np.testing.assert_allclose(got[0, 0, k], brute.norm_row(rows[0, 0, k].tolist()), rtol=1e-15)


# ---------------------------------------------------------------------------
# a1: pooling
# ---------------------------------------------------------------------------
def test_pool_golden_2x2(golden_dir):
    g = read_golden(os.path.join(golden_dir, "pool_2x2.txt"))
    h, w, C = int(g["h"][0]), int(g["w"][0]), int(g["C"][0])
    sigma = math.sqrt(float(g["sigma2_times_ln2"][0]) / math.log(2.0))
    S = np.zeros((1, h, w, C))
    for i in range(h):
        for j in range(w):
            S[0, i, j] = list(map(float, g[f"F{i}{j}"]))
    kp = np.array([[[float(g["x"][0]), float(g["y"][0])]]])
    proto = O.pool_prototypes(S, kp, np.ones((1, 1), np.uint8), sigma, float(g["stride"][0]))
    want = np.array(list(map(float, g["expected_num"]))) / float(g["expected_den"][0])
    np.testing.assert_allclose(proto[0, 0], want, rtol=1e-14)


def test_pool_constant_map_gives_constant():
    S = np.full((2, 24, 24, 5), -2.5)
    kp = RNG.uniform(0, 384, size=(2, 7, 2))
    proto = O.pool_prototypes(S, kp, np.ones((2, 7), np.uint8), 14.0, 16.0)
    np.testing.assert_allclose(proto, -2.5, rtol=1e-14)


def test_pool_small_sigma_picks_nearest_patch():
    S = RNG.standard_normal((1, 24, 24, 6))
    kp = np.array([[[16 * 3 + 8, 16 * 17 + 8],      # exactly at patch (17, 3)
                    [16 * 20 + 8.3, 16 * 2 + 7.1]]])  # near patch (2, 20)
    proto = O.pool_prototypes(S, kp, np.ones((1, 2), np.uint8), 0.1, 16.0)
    np.testing.assert_array_equal(proto[0, 0], S[0, 17, 3])
    np.testing.assert_array_equal(proto[0, 1], S[0, 2, 20])


def test_pool_mirror_symmetry():
    S = RNG.standard_normal((1, 24, 24, 4))
    Sm = S[:, :, ::-1].copy()                      # mirror in x
    x, y = 101.3, 250.9
    a = O.pool_prototypes(S, np.array([[[x, y]]]), np.ones((1, 1), np.uint8), 14.0, 16.0)
    b = O.pool_prototypes(Sm, np.array([[[384.0 - x, y]]]), np.ones((1, 1), np.uint8), 14.0, 16.0)
    np.testing.assert_allclose(a, b, rtol=1e-13)


def test_pool_matches_brute_force_and_masks():
    B, h, w, C, K = 2, 3, 4, 5, 3
    S = RNG.standard_normal((B, h, w, C))
    kp = RNG.uniform(0, 64, size=(B, K, 2))
    km = np.array([[1, 0, 1], [0, 1, 1]], np.uint8)
    proto = O.pool_prototypes(S, kp, km, 9.0, 16.0)
    for b in range(B):
        for k in range(K):
            if not km[b, k]:
                assert np.all(proto[b, k] == 0)
                continue
            ref = brute.pool_row(S[b].tolist(), h, w, C, kp[b, k, 0], kp[b, k, 1], 9.0, 16.0)
            np.testing.assert_allclose(proto[b, k], ref, rtol=1e-13)


# ---------------------------------------------------------------------------
# a5 + a6: fusion and decode
# ---------------------------------------------------------------------------
def test_decode_xy_golden(golden_dir):
    path = os.path.join(golden_dir, "decode_xy.txt")
    with open(path) as f:
        lines = [l.split() for l in f if l.strip() and not l.startswith("#")]
    for W_s, col_s, num_s, den_s in lines:
        W, col = int(W_s), int(col_s)
        heat = np.zeros((1, 1, 1, 1, W), np.float32)
        heat[..., col] = 1.0
        _, idx, xy, _, _ = O.fuse_decode(heat.reshape(1, 1, 1, 1, W), np.ones((1, 1, 1), np.uint8))
        assert idx[0, 0] == col
        want = f32_from_fraction(Fraction(int(num_s), int(den_s)))
        assert xy[0, 0, 0] == want, (W, col)


def test_decode_xy_2d_golden(golden_dir):
    """Row-major index and both coordinates on square, wide, tall and ragged grids."""
    path = os.path.join(golden_dir, "decode_xy2d.txt")
    with open(path) as f:
        lines = [[int(v) for v in l.split()] for l in f if l.strip() and not l.startswith("#")]
    for H, W, row, col, index, xn, xd, yn, yd in lines:
        heat = np.zeros((1, 1, 1, H, W), np.float32)
        heat[0, 0, 0, row, col] = 2.0
        _, idx, xy, score, valid = O.fuse_decode(heat, np.ones((1, 1, 1), np.uint8))
        assert idx[0, 0] == index == row * W + col
        assert xy[0, 0, 0] == f32_from_fraction(Fraction(xn, xd)), (H, W, "x")
        assert xy[0, 0, 1] == f32_from_fraction(Fraction(yn, yd)), (H, W, "y")
        assert score[0, 0] == 2.0 and valid[0, 0] == 1


def test_decode_matches_torch_argmax_and_brute():
    heat = RNG.standard_normal((2, 2, 3, 8, 12)).astype(np.float32)
    heat[0, 0, 1, 2, 3] = heat[0, 0, 1, 5, 1] = 7.0       # tie inside one modality
    mask = np.array([[[1, 1, 0], [0, 1, 0]], [[1, 0, 1], [1, 1, 1]]], np.uint8)
    fused, idx, xy, score, valid = O.fuse_decode(heat, mask)
    for b in range(2):
        for k in range(3):
            pres = [m for m in range(2) if mask[b, m, k]]
            if not pres:
                assert (idx[b, k], valid[b, k], score[b, k]) == (-1, 0, 0)
                assert np.all(xy[b, k] == 0)
                continue
            if len(pres) == 2:
                f = (heat[b, 0, k] + heat[b, 1, k]) * np.float32(0.5)
            else:
                f = heat[b, pres[0], k]
            np.testing.assert_array_equal(fused[b, k], f)
            t = int(torch.argmax(torch.from_numpy(f.reshape(-1))))
            assert idx[b, k] == t == brute.argmax_first(f.reshape(-1).tolist())
            assert score[b, k] == f.reshape(-1)[t]
            assert valid[b, k] == 1
    assert idx[0, 1] == 2 * 12 + 3 or mask[0, 1, 1] == 1


def test_decode_first_index_on_ties_and_signed_zero():
    heat = np.full((1, 1, 1, 4, 4), -1.0, np.float32)
    heat[0, 0, 0, 1, 2] = -0.0
    heat[0, 0, 0, 0, 3] = 0.0
    heat[0, 0, 0, 3, 3] = 0.0
    _, idx, _, score, _ = O.fuse_decode(heat, np.ones((1, 1, 1), np.uint8))
    assert idx[0, 0] == 3 and score[0, 0] == 0.0


def test_decode_xy_is_antisymmetric():
    W = 96
    xs = []
    for col in range(W):
        heat = np.zeros((1, 1, 1, 1, W), np.float32)
        heat[..., col] = 1.0
        xs.append(O.fuse_decode(heat, np.ones((1, 1, 1), np.uint8))[2][0, 0, 0])
    for col in range(W):
        assert xs[col] == -xs[W - 1 - col]
        assert xs[col] == np.float32((2 * col + 1 - W) / W)


def test_planted_peak_is_recovered():
    """A Gaussian bump of width 1 patch planted at (u, v) (patch units) along a
    unit direction, matched with that direction: the decoded peak lies within
    2.5 heatmap pixels of 4u - 0.5 (the bilinear interpolant of a peaked
    function is maximal at a source node within half a patch of (u, v), and its
    output samples sit 1/8 patch from the node)."""
    C, h, w = 32, 24, 24
    rng = np.random.default_rng(7)
    for trial in range(20):
        d = rng.standard_normal(C)
        d /= np.linalg.norm(d)
        u, v = rng.uniform(0.5, 23.5, size=2)
        jj = np.arange(w) + 0.5
        ii = np.arange(h) + 0.5
        g = np.exp(-0.5 * ((jj[None, :] - u) ** 2 + (ii[:, None] - v) ** 2))
        F = 4.0 * g[:, :, None] * d[None, None, :]
        heat = O.heatmap_crop(F, d[None, None, :], np.ones((1, 1), np.uint8), 4, "f32")
        _, idx, xy, score, _ = O.fuse_decode(heat[None].astype(np.float32), np.ones((1, 1, 1), np.uint8))
        p = int(idx[0, 0])
        assert abs(p % 96 - (4 * u - 0.5)) <= 2.5 and abs(p // 96 - (4 * v - 0.5)) <= 2.5
        assert score[0, 0] > 4.0 * 0.765625 * math.exp(-0.25) - 1e-6


def test_head_chain_consistency_small():
    """The full oracle chain equals its steps composed by hand."""
    B, h, w, C, K = 2, 3, 3, 16, 4
    feat = RNG.standard_normal((B, h, w, C))
    rows = RNG.standard_normal((B, 2, K, C))
    mask = (RNG.random((B, 2, K)) < 0.6).astype(np.uint8)
    heat, (fused, idx, xy, score, valid) = O.head(feat, rows, mask, operand="bf16")
    kh = O.bf16_round(O.norm_rows(rows, mask))
    for b in range(B):
        U = O.bf16_round(O.upsample(feat[b]))
        for m in range(2):
            for k in range(K):
                if mask[b, m, k]:
                    np.testing.assert_allclose(heat[b, m, k], U @ kh[b, m, k], rtol=1e-12)
    assert np.array_equal(valid, (mask.sum(1) > 0).astype(np.uint8))


def test_out_rows_selection_is_a_restriction():
    F = RNG.standard_normal((5, 6, 3))
    kern = RNG.standard_normal((2, 2, 3))
    mask = np.ones((2, 2), np.uint8)
    full = O.heatmap_crop(F, kern, mask, 4, "bf16")
    part = O.heatmap_crop(F, kern, mask, 4, "bf16", out_rows=[3, 0, 17])
    np.testing.assert_array_equal(part, full[:, :, [3, 0, 17]])
