"""Pins of the variant oracles (fusion by linearity, contract then upsample,
ROI -> image coordinates) to facts other than themselves (CPU only).

Each variant is tied to the graded oracle by the linearity identity it rests
on (float64, no rounding), to closed forms on one-hot and constant maps, to
the pure-Python brute force on tiny inputs, and, for the coordinate map, to
its fixed points, an independent composition of the resize and pad as
homogeneous matrices, and the bounding-box example of the model card.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from conftest import read_golden
from oracle import brute
from oracle import gkd_oracle as O
from oracle import variants as V

RNG = np.random.default_rng(2024)


def _brute_bf16(x: float) -> float:
    """Independent fp64 -> bf16 rounding (frexp + Python's half-even round)."""
    if x == 0.0 or not math.isfinite(x):
        return x
    m, e = math.frexp(x)
    q = math.ldexp(1.0, max(e - 8, -133))
    return round(x / q) * q


def _mask_all_cases(Bk, K):
    """[Bk][2][K] masks holding every (visual, text) combination, plus random rows."""
    m = (RNG.random((Bk, 2, K)) < 0.6).astype(np.uint8)
    for b in range(Bk):
        m[b, :, 0] = (1, 1)
        m[b, :, 1] = (1, 0)
        m[b, :, 2] = (0, 1)
        m[b, :, 3] = (0, 0)
    return m


# ---------------------------------------------------------------------------
# fusion by linearity
# ---------------------------------------------------------------------------
def test_fused_kernels_equal_mean_of_heatmaps_f64():
    B, h, w, C, K = 3, 5, 6, 16, 7
    feat = RNG.standard_normal((B, h, w, C))
    rows = RNG.standard_normal((B, 2, K, C))
    mask = _mask_all_cases(B, K)
    _, (fused, idx, xy, score, valid) = O.head(feat, rows, mask, operand="f32")
    heat_f, (_, idx_f, xy_f, score_f, valid_f) = V.head_fused_kernels(feat, rows, mask, operand="f32")
    np.testing.assert_array_equal(valid_f, valid)
    assert valid.sum() > 0 and (valid == 0).sum() > 0
    for b in range(B):
        for k in range(K):
            if not valid[b, k]:
                assert np.all(np.isnan(heat_f[b, k])) and idx_f[b, k] == -1
                continue
            ref = fused[b, k]
            np.testing.assert_allclose(heat_f[b, k], ref, rtol=0, atol=1e-12 * np.abs(ref).max())
            if O.top2_margin(ref) > 1e-9 * np.abs(ref).max():
                assert idx_f[b, k] == idx[b, k]
                np.testing.assert_array_equal(xy_f[b, k], xy[b, k])


@pytest.mark.parametrize("operand", ["f32", "bf16"])
def test_fused_kernels_single_modality_rows_equal_graded(operand):
    B, h, w, C, K = 2, 4, 5, 8, 6
    feat = RNG.standard_normal((B, h, w, C))
    if operand == "bf16":
        feat = O.bf16_round(feat)
    rows = RNG.standard_normal((B, 2, K, C))
    mask = _mask_all_cases(B, K)
    heat, _ = O.head(feat, rows, mask, operand=operand)
    heat_f, _ = V.head_fused_kernels(feat, rows, mask, operand=operand)
    n = 0
    for b in range(B):
        for k in range(K):
            present = [m for m in range(2) if mask[b, m, k]]
            if len(present) == 1:
                np.testing.assert_array_equal(heat_f[b, k], heat[b, present[0], k])
                n += 1
    assert n >= 2 * B


@pytest.mark.parametrize("operand", ["f32", "bf16"])
def test_fused_kernels_onehot_closed_form(operand):
    # feature e_c at interior cell (2, 3); visual row e_c, text row e_d: the fused
    # row is (e_c + e_d) / 2, so the heatmap is U_c / 2 with peak (7/8)^2 / 2 at the
    # 2x2 block starting at (4*2+1, 4*3+1); the first of the tie is decoded.
    h, w, C, c, d = 6, 6, 8, 2, 5
    feat = np.zeros((1, h, w, C))
    feat[0, 2, 3, c] = 1.0
    rows = np.zeros((1, 2, 1, C))
    rows[0, 0, 0, c] = 3.0
    rows[0, 1, 0, d] = 0.25
    mask = np.ones((1, 2, 1), np.uint8)
    heat_f, (_, idx, xy, score, valid) = V.head_fused_kernels(feat, rows, mask, operand=operand)
    peak = 0.765625 / 2
    assert heat_f.max() == peak
    Y, X = np.nonzero(heat_f[0, 0] == peak)
    assert sorted(zip(Y.tolist(), X.tolist())) == [(9, 13), (9, 14), (10, 13), (10, 14)]
    W = 4 * w
    assert idx[0, 0] == 9 * W + 13 and score[0, 0] == np.float32(peak) and valid[0, 0] == 1
    assert xy[0, 0, 0] == np.float32(27 - W) / np.float32(W)
    assert xy[0, 0, 1] == np.float32(19 - W) / np.float32(W)


@pytest.mark.parametrize("operand", ["f32", "bf16"])
def test_fused_kernels_match_brute_force_tiny(operand):
    rnd = _brute_bf16 if operand == "bf16" else None
    for trial in range(5):
        h, w = int(RNG.integers(1, 4)), int(RNG.integers(1, 4))
        C, K = int(RNG.integers(1, 7)), 4
        feat = RNG.standard_normal((1, h, w, C))
        rows = RNG.standard_normal((1, 2, K, C))
        mask = _mask_all_cases(1, K)
        heat_f, _ = V.head_fused_kernels(feat, rows, mask, operand=operand)
        Fl = feat[0].tolist()
        for k in range(K):
            present = [m for m in range(2) if mask[0, m, k]]
            if not present:
                assert np.all(np.isnan(heat_f[0, k]))
                continue
            kr = brute.mean_row([brute.norm_row(rows[0, m, k].tolist()) for m in present])
            if rnd is not None:
                kr = [rnd(v) for v in kr]
            for Y in range(4 * h):
                for X in range(4 * w):
                    ref = brute.heat_value(Fl, h, w, C, kr, Y, X, 4, rnd)
                    assert abs(heat_f[0, k, Y, X] - ref) <= 1e-12 * max(1.0, abs(ref))


def test_fused_kernel_rows_round_once_after_the_mean():
    # 1 + 2^-8 is a bf16 tie (rounds down to 1) and 1 + 2^-7 + 2^-9 rounds to
    # 1 + 2^-7; their exact mean 1 + 7/1024 rounds up to 1 + 2^-7. Rounding the
    # rows before the mean would give 1 + 2^-8 instead
    a = np.array([1.0 + 2.0 ** -8])                  # not a bf16 value (needs 9 bits)
    b = np.array([1.0 + 2.0 ** -7 + 2.0 ** -9])
    khat = np.stack([a, b])[None, :, None, :]        # [1][2][1][1]
    kf, valid = V.fused_kernel_rows(khat, np.ones((1, 2, 1), np.uint8), "bf16")
    exact = (a[0] + b[0]) / 2                          # 1 + 7/1024
    assert kf[0, 0, 0] == O.bf16_round(np.array([exact]))[0] == 1.0078125
    first_rounded = (O.bf16_round(a)[0] + O.bf16_round(b)[0]) / 2
    assert first_rounded != kf[0, 0, 0]


# ---------------------------------------------------------------------------
# contract then upsample
# ---------------------------------------------------------------------------
def test_contract_first_equals_graded_f64():
    h, w, C, M, K = 7, 5, 24, 2, 4
    F = RNG.standard_normal((h, w, C))
    kern = RNG.standard_normal((M, K, C))
    mask = (RNG.random((M, K)) < 0.7).astype(np.uint8)
    mask[0, 0] = 1
    mask[1, 0] = 0
    a = V.heatmap_crop_contract_first(F, kern, mask, 4, "f32")
    b = O.heatmap_crop(F, kern, mask, 4, "f32")
    np.testing.assert_array_equal(np.isnan(a), np.isnan(b))
    for m in range(M):
        for k in range(K):
            if mask[m, k]:
                np.testing.assert_allclose(a[m, k], b[m, k], rtol=0, atol=1e-12 * np.abs(b[m, k]).max())


def test_contract_first_constant_map_exact():
    # constant bf16-exact feature vector v and bf16-exact rows: every heatmap value
    # is exactly sum_c k_c v_c (dyadic values, exact in float64)
    C, K = 16, 3
    v = RNG.integers(-128, 128, C) / 64.0
    kern = (RNG.integers(-128, 128, (1, K, C)) / 64.0)
    F = np.broadcast_to(v, (4, 5, C)).copy()
    heat = V.heatmap_crop_contract_first(F, kern, np.ones((1, K), np.uint8), 4, "bf16")
    for k in range(K):
        exact = sum(Fraction(float(kern[0, k, c])) * Fraction(float(v[c])) for c in range(C))
        assert np.all(heat[0, k] == float(exact))


def test_contract_first_onehot_closed_form():
    h, w, C = 5, 7, 4
    F = np.zeros((h, w, C))
    F[1, 4, 3] = 1.0
    kern = np.zeros((1, 1, C))
    kern[0, 0, 3] = 1.0
    heat = V.heatmap_crop_contract_first(F, kern, np.ones((1, 1), np.uint8), 4, "bf16")
    assert heat.max() == 0.765625
    Y, X = np.nonzero(heat[0, 0] == 0.765625)
    assert sorted(zip(Y.tolist(), X.tolist())) == [(5, 17), (5, 18), (6, 17), (6, 18)]
    # the corner cell reaches 1.0 on the clamped 2x2 block at the origin
    F2 = np.zeros((h, w, C))
    F2[0, 0, 3] = 1.0
    heat2 = V.heatmap_crop_contract_first(F2, kern, np.ones((1, 1), np.uint8), 4, "f32")
    assert heat2[0, 0, :2, :2].tolist() == [[1.0, 1.0], [1.0, 1.0]] and heat2.max() == 1.0


@pytest.mark.parametrize("operand", ["f32", "bf16"])
def test_contract_first_matches_brute_force_tiny(operand):
    rnd = _brute_bf16 if operand == "bf16" else None
    for trial in range(5):
        h, w = int(RNG.integers(1, 5)), int(RNG.integers(1, 5))
        C, K = int(RNG.integers(1, 9)), int(RNG.integers(1, 4))
        F = RNG.standard_normal((h, w, C))
        kern = RNG.standard_normal((1, K, C))
        heat = V.heatmap_crop_contract_first(F, kern, np.ones((1, K), np.uint8), 4, operand)
        Fl = F.tolist()
        for k in range(K):
            for Y in range(4 * h):
                for X in range(4 * w):
                    ref = brute.contract_first_value(Fl, h, w, C, kern[0, k].tolist(), Y, X, 4, rnd)
                    assert abs(heat[0, k, Y, X] - ref) <= 1e-12 * max(1.0, abs(ref))


def test_contract_first_head_decodes_like_graded_f64():
    B, h, w, C, K = 2, 6, 6, 32, 5
    feat = RNG.standard_normal((B, h, w, C))
    rows = RNG.standard_normal((B, 2, K, C))
    mask = _mask_all_cases(B, K)
    _, (fused, idx, xy, score, valid) = O.head(feat, rows, mask, operand="f32")
    _, (fused_c, idx_c, xy_c, score_c, valid_c) = V.head_contract_first(feat, rows, mask, operand="f32")
    np.testing.assert_array_equal(valid_c, valid)
    for b in range(B):
        for k in range(K):
            if valid[b, k] and O.top2_margin(fused[b, k]) > 1e-9 * np.abs(fused[b, k]).max():
                assert idx_c[b, k] == idx[b, k]
                assert abs(float(score_c[b, k]) - float(score[b, k])) <= 1e-6 * abs(float(score[b, k])) + 1e-30


# ---------------------------------------------------------------------------
# ROI -> image coordinates
# ---------------------------------------------------------------------------
BOXES = [(33, 38, 241, 310), (0, 0, 640, 480), (10.5, 20.25, 110.5, 70.25), (5, 5, 105, 105)]


@pytest.mark.parametrize("box", BOXES)
def test_roi_centre_and_longer_side_ends(box):
    x0, y0, x1, y1 = box
    bw, bh = x1 - x0, y1 - y0
    cx, cy = (x0 + x1) / 2, (y0 + y1) / 2
    L = max(bw, bh)
    pts = V.roi_to_image(np.array([[0.0, 0.0], [-1.0, -1.0], [1.0, 1.0]]), box)
    assert np.allclose(pts[0], (cx, cy), rtol=0, atol=1e-12 * L)
    # the canvas spans the longer side exactly and is centred on the box on both axes
    assert np.allclose(pts[1], (cx - L / 2, cy - L / 2), rtol=0, atol=1e-12 * L)
    assert np.allclose(pts[2], (cx + L / 2, cy + L / 2), rtol=0, atol=1e-12 * L)
    if bh >= bw:
        assert abs(pts[1, 1] - y0) <= 1e-12 * L and abs(pts[2, 1] - y1) <= 1e-12 * L
    if bw >= bh:
        assert abs(pts[1, 0] - x0) <= 1e-12 * L and abs(pts[2, 0] - x1) <= 1e-12 * L


def _homogeneous_forward(box, canvas=384):
    """Original pixel -> normalised ROI coordinate, composed as 3x3 matrices:
    translate the box origin to 0, scale by canvas / longer side, translate by
    the centred pad, then map canvas pixels [0, canvas] onto [-1, 1]."""
    x0, y0, x1, y1 = box
    bw, bh = x1 - x0, y1 - y0
    s = canvas / max(bw, bh)
    T0 = np.array([[1, 0, -x0], [0, 1, -y0], [0, 0, 1]], float)
    S = np.diag([s, s, 1.0])
    P = np.array([[1, 0, (canvas - s * bw) / 2], [0, 1, (canvas - s * bh) / 2], [0, 0, 1]], float)
    N = np.array([[2 / canvas, 0, -1], [0, 2 / canvas, -1], [0, 0, 1]], float)
    return N @ P @ S @ T0


@pytest.mark.parametrize("box", BOXES)
def test_roi_map_inverts_the_composed_preprocessing(box):
    A = _homogeneous_forward(box)
    u = RNG.uniform(-1, 1, (50, 2))
    pts = V.roi_to_image(u, box)
    back = (A @ np.c_[pts, np.ones(len(pts))].T).T[:, :2]
    np.testing.assert_allclose(back, u, rtol=0, atol=1e-12)
    np.testing.assert_allclose(V.image_to_roi(pts, box), u, rtol=0, atol=1e-12)


def test_roi_grid_cells_land_on_canvas_cell_centres():
    W = 96
    cols = np.arange(W)
    u = (2 * cols + 1 - W) / W
    canvas_px = (u + 1) * 384 / 2
    # exact in real arithmetic; u itself is rounded (96 is not a power of two)
    np.testing.assert_allclose(canvas_px, 4 * (cols + 0.5), rtol=0, atol=1e-12)
    # with a box equal to the canvas, ROI pixels are canvas pixels
    pts = V.roi_to_image(np.stack([u, u], -1), (0, 0, 384, 384))
    np.testing.assert_allclose(pts, np.stack([4 * (cols + 0.5)] * 2, -1), rtol=0, atol=1e-12)


def test_roi_cell_size_matches_the_model_card_box(golden_dir):
    g = read_golden(f"{golden_dir}/roi_box.txt")
    box = tuple(float(v) for v in g["box"])
    err = float(g["near_tie_error_px"][0])
    G = int(g["grid"][0])
    a = V.roi_to_image(np.array([[0.0, 0.0], [2.0 / G, 0.0], [0.0, 2.0 / G]]), box)
    step_x, step_y = a[1, 0] - a[0, 0], a[2, 1] - a[0, 1]
    assert abs(step_x - 272 / 96) <= 1e-12 and abs(step_y - 272 / 96) <= 1e-12
    # one grid cell of that box is within 1% of the card's near-tie error figure
    assert abs(step_y - err) / err < 0.01


def test_roi_rejects_degenerate_boxes():
    for box in [(0, 0, 0, 10), (5, 5, 5, 5), (10, 0, 0, 10)]:
        with pytest.raises(ValueError):
            V.roi_to_image(np.zeros((1, 2)), box)
